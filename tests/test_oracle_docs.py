"""Every public function of the oracle says which source passage (or format definition) it
follows, and the oracle's modules keep their test-infrastructure header."""
import ast
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
MODULES = ["oracle/numerics.py", "oracle/vit.py", "oracle/perturb.py"]
CITE = re.compile(r"\[(?:FRT|VE|TRT)\b[^\]]*\]|OCP E4M3|bfloat16 format")


@pytest.mark.parametrize("path", MODULES)
def test_oracle_functions_cite_their_source(path):
    tree = ast.parse(open(os.path.join(ROOT, path)).read())
    assert "TEST INFRASTRUCTURE ONLY" in (ast.get_docstring(tree) or "")
    missing = [n.name for n in tree.body
               if isinstance(n, ast.FunctionDef) and not n.name.startswith("_")
               and not CITE.search(ast.get_docstring(n) or "")]
    assert not missing, missing
