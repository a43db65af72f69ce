// vit_merger_forward_static: the 2x2 merger with its scratch in a fixed
// device array of this library instead of a caller-supplied workspace.
//
// Some callers cannot hand the library a workspace: code running inside an
// allocator callback or a plugin host that forbids device allocations after
// start-up, or a serving loop that must never call cudaMalloc (it can
// synchronise the device and stall other streams).  This entry point needs no
// allocation at all: its intermediates (FP8 codes, scales, fc1 output) live in
// g_merger_scratch below, whose device address is looked up once per device.
#include <mutex>

namespace vitq {
namespace {

constexpr size_t up256c(size_t b) { return (b + 255) & ~size_t(255); }
constexpr size_t kStaticMergerRows = VITQ_MERGER_STATIC_MAX_TOKENS / 4;
// Same layout as the workspace of vit_merger_forward for the largest input:
// codes [rows, 4608] u8, scales [36, rows] fp32, fc1 output [rows, 4608] bf16.
constexpr size_t kStaticMergerBytes = up256c(kStaticMergerRows * VITQ_MERGE_IN) +
                                      up256c((VITQ_MERGE_IN / 128) * ((kStaticMergerRows + 3) & ~size_t(3)) * 4) +
                                      up256c(kStaticMergerRows * VITQ_MERGE_IN * 2);

}  // namespace

// One array per device, shared by every call on that device.  No byte of it
// has to start at zero: each call writes every scratch byte before reading it.
static __device__ __align__(256) uint8_t g_merger_scratch[kStaticMergerBytes];

namespace {

uint8_t* g_merger_scratch_ptr[kMaxDevices] = {};
std::mutex g_merger_scratch_mu;

// Device address of g_merger_scratch on the current device (looked up on the
// first call per device, which may also load this library's kernels there).
int merger_scratch_on_current_device(uint8_t** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return VITQ_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_merger_scratch_mu);
  if (!g_merger_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_merger_scratch) != cudaSuccess || !p) return VITQ_ERR_CUDA;
    g_merger_scratch_ptr[dev] = reinterpret_cast<uint8_t*>(p);
  }
  *out = g_merger_scratch_ptr[dev];
  return VITQ_OK;
}

}  // namespace
}  // namespace vitq

extern "C" int vit_merger_forward_static(const vitq_merger_weights* w, const void* x, int n_tokens, void* out,
                                         void* stream) {
  using namespace vitq;
  VITQ_CHECK(merger_weights_ok(w), w ? VITQ_ERR_ALIGN : VITQ_ERR_INVALID_ARG);
  VITQ_CHECK(x && out && n_tokens >= 0, VITQ_ERR_INVALID_ARG);
  VITQ_CHECK(n_tokens % 4 == 0, VITQ_ERR_SHAPE);
  VITQ_CHECK(al16(x) && al16(out), VITQ_ERR_ALIGN);
  VITQ_CHECK(n_tokens <= VITQ_MERGER_STATIC_MAX_TOKENS &&
                 vitq_merger_workspace_bytes(n_tokens) <= sizeof(g_merger_scratch),
             VITQ_ERR_WORKSPACE);
  int sms = 0;
  int r = current_device_ok(&sms);
  if (r) return r;
  uint8_t* scratch = nullptr;
  r = merger_scratch_on_current_device(&scratch);
  if (r) return r;
  if (n_tokens == 0) return VITQ_OK;
  Carver c{scratch};
  MergerWs m = carve_merger(c, n_tokens);
  return merger_impl(w, (const __nv_bfloat16*)x, n_tokens, (__nv_bfloat16*)out, m, sms, reinterpret_cast<cudaStream_t>(stream));
}
