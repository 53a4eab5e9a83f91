"""Every kernel the library launches with programmatic stream serialization
(``launch_chained``) may start while the kernel before it on the stream is
still running, so it must wait on the device (``grid_dep_wait()``) before it
touches global memory.  This host-side check reads the CUDA sources: each
kernel named in a ``launch_chained(...)`` call is defined in the same file and
its body calls ``grid_dep_wait()``; a kernel that also holds tensor memory
triggers its dependents (``grid_dep_launch()``) only after its allocation."""

import os
import re

CSRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "block_sparse_attention_psa_b200",
                    "csrc")


def _kernel_body(src, name):
    m = re.search(r"__global__[^{;]*?\b" + re.escape(name) + r"\s*\(", src)
    assert m, f"kernel {name} is not defined where it is launched"
    i = src.index("{", m.end())
    depth = 0
    for j in range(i, len(src)):
        depth += {"{": 1, "}": -1}.get(src[j], 0)
        if depth == 0:
            return src[i:j + 1]
    raise AssertionError(f"unbalanced body of {name}")


def test_every_chained_kernel_waits_before_global_memory():
    seen = 0
    for f in sorted(os.listdir(CSRC)):
        if not f.endswith(".cu"):
            continue
        src = open(os.path.join(CSRC, f)).read()
        for name in sorted(set(re.findall(r"launch_chained\(\s*([A-Za-z_]\w*)", src))):
            body = _kernel_body(src, name)
            assert "grid_dep_wait()" in body, f"{f}: {name} is chained but never waits"
            if "tmem_alloc(" in body:
                assert body.index("tmem_alloc(") < body.index("grid_dep_launch()"), \
                    f"{f}: {name} triggers its dependents before its tensor-memory allocation"
            seen += 1
    assert seen >= 10
