"""The key of the stored profiler records: the code of the kernel's sources, not their comments."""
from tree_routed_sparse_b200 import build


def test_code_only_ignores_comments_and_blank_lines():
    a = "int f() { return 1; }  // one\n/* a block\n   comment */\n\n"
    b = "// a comment first\nint f() { return 1; }\n"
    c = "int f() { return 2; }\n"
    assert build.code_only(a) == build.code_only(b) == "int f() { return 1; }"
    assert build.code_only(a) != build.code_only(c)


def test_kernel_hash_is_stable_and_per_file():
    h = build.kernel_hash("query_kernels.cu")
    assert h == build.kernel_hash("query_kernels.cu") and len(h) == 40
    assert h != build.kernel_hash("label_kernels.cu")
