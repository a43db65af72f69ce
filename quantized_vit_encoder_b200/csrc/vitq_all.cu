// Single translation unit for libvitq.so (the kernels share one device error word).
#include "elementwise.cu"
#include "gemm_fp8.cu"
#include "gemm_bf16.cu"
#include "attention.cu"
#include "api.cu"
#include "merger_static.cu"
