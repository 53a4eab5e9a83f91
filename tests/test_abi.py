"""CPU checks of the C-ABI library: it loads, exports every entry point that
include/psa.h declares, and rejects bad arguments on the host (these calls
return before any CUDA call, so they need no GPU)."""

import ctypes
import os
import re

import pytest

from block_sparse_attention_psa_b200 import psa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
FAKE = ctypes.c_void_p(1 << 20)   # a 16-byte-aligned address that is never dereferenced


def declared_symbols():
    with open(os.path.join(ROOT, "include", "psa.h")) as f:
        text = f.read()
    return sorted(set(re.findall(r"PSA_API\s+[\w\s\*]*?\b(psa_\w+)\s*\(", text)))


def test_header_declares_the_path():
    names = declared_symbols()
    for want in ("psa_pool", "psa_route_topk", "psa_route_thresh", "psa_attn", "psa_dense"):
        assert want in names


def test_library_exports_every_declared_symbol():
    L = psa.lib()
    names = declared_symbols()
    assert names
    for name in names:
        assert hasattr(L, name), name
    assert set(psa.EXPORTS) == set(names)


def test_status_strings():
    for code in range(0, 9):
        assert psa.status_text(code)
    assert psa.status_text(PSA_UNKNOWN := 1234) == "unknown status"


def test_workspace_and_capacity_sizes():
    assert psa.psa_workspace_size(1, 12, 32768, 128) > 0
    assert psa.psa_workspace_size(1, 12, 32768 + 1, 128) == 0      # ragged N
    assert psa.psa_workspace_size(1, 12, 32768, 96) == 0            # unsupported d
    assert psa.psa_route_capacity(1, 12, 512, False) == 12 * 512 * 512
    assert psa.psa_route_capacity(1, 8, 2048, True) == 8 * 2048 * 2049 // 2
    assert psa.psa_route_capacity(0, 8, 2048, True) == 0


def test_host_validation_rejects_bad_arguments():
    L = psa.lib()
    S = ctypes.c_void_p(0)
    # null pointers
    assert L.psa_pool(None, FAKE, FAKE, 1, 1, 64, 64, 64, FAKE, FAKE, FAKE, S) == psa.PSA_ERR_ARG
    # block size, head dim, ragged N
    assert L.psa_pool(FAKE, FAKE, FAKE, 1, 1, 64, 64, 32, FAKE, FAKE, FAKE, S) == psa.PSA_ERR_UNSUPPORTED
    assert L.psa_pool(FAKE, FAKE, FAKE, 1, 1, 64, 80, 64, FAKE, FAKE, FAKE, S) == psa.PSA_ERR_UNSUPPORTED
    assert L.psa_pool(FAKE, FAKE, FAKE, 1, 1, 100, 64, 64, FAKE, FAKE, FAKE, S) == psa.PSA_ERR_SHAPE
    assert L.psa_pool(FAKE, FAKE, FAKE, 0, 1, 64, 64, 64, FAKE, FAKE, FAKE, S) == psa.PSA_ERR_ARG
    # misaligned tensor
    assert L.psa_pool(ctypes.c_void_p((1 << 20) + 2), FAKE, FAKE, 1, 1, 64, 64, 64, FAKE, FAKE, FAKE, S) \
        == psa.PSA_ERR_ARG
    # top-k: capacity below the exact total, bad density
    big = 1 << 40
    assert L.psa_route_topk(FAKE, FAKE, 1, 2, 16, 64, 0.25, 0, FAKE, FAKE, 2 * 16 * 4 - 1, FAKE, None, FAKE, big,
                            S) == psa.PSA_ERR_CAPACITY
    assert L.psa_route_topk(FAKE, FAKE, 1, 2, 16, 64, float("nan"), 0, FAKE, FAKE, 1 << 20, FAKE, None, FAKE, big,
                            S) == psa.PSA_ERR_ARG
    assert L.psa_route_topk(FAKE, FAKE, 1, 2, 16, 64, 0.25, 2, FAKE, FAKE, 1 << 20, FAKE, None, FAKE, big, S) \
        == psa.PSA_ERR_ARG
    # top-k: workspace missing, misaligned, too small
    assert L.psa_route_topk(FAKE, FAKE, 1, 2, 16, 64, 0.25, 0, FAKE, FAKE, 1 << 20, FAKE, None, None, big, S) \
        == psa.PSA_ERR_ARG
    assert L.psa_route_topk(FAKE, FAKE, 1, 2, 16, 64, 0.25, 0, FAKE, FAKE, 1 << 20, FAKE, None,
                            ctypes.c_void_p((1 << 20) + 16), big, S) == psa.PSA_ERR_ARG
    need = psa.psa_workspace_size(1, 2, 16 * 64, 64)
    assert L.psa_route_topk(FAKE, FAKE, 1, 2, 16, 64, 0.25, 0, FAKE, FAKE, 1 << 20, FAKE, None, FAKE, need - 1,
                            S) == psa.PSA_ERR_CAPACITY
    # threshold: workspace too small, bad alpha
    assert L.psa_route_thresh(FAKE, FAKE, 1, 2, 16, 64, 0.5, 0, 0, FAKE, FAKE, 1 << 20, FAKE, None, FAKE, 16, S) \
        == psa.PSA_ERR_CAPACITY
    assert L.psa_route_thresh(FAKE, FAKE, 1, 2, 16, 64, float("inf"), 0, 0, FAKE, FAKE, 1 << 20, FAKE, None,
                              FAKE, 1 << 30, S) == psa.PSA_ERR_ARG
    # attention: workspace too small, misaligned workspace, M too large
    ws = psa.psa_workspace_size(1, 2, 1024, 64)
    assert L.psa_attn(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 64, None, 1, 2, 1024, 64, 64, 0, FAKE, None,
                      FAKE, ws - 1, S) == psa.PSA_ERR_CAPACITY
    assert L.psa_attn(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 64, None, 1, 2, 1024, 64, 64, 0, FAKE,
                      None, ctypes.c_void_p((1 << 20) + 16), ws, S) == psa.PSA_ERR_ARG
    assert L.psa_attn(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 64, None, 1, 1, 64 * 16385, 64, 64, 0, FAKE,
                      None, FAKE, 1 << 40, S) == psa.PSA_ERR_UNSUPPORTED
    # probability-domain threshold: alpha must be positive and finite
    for bad_alpha in (0.0, -0.5, float("nan"), float("inf")):
        assert L.psa_route_thresh_prob(FAKE, FAKE, 1, 2, 16, 64, bad_alpha, 0, 0, FAKE, FAKE, 1 << 20, FAKE, None,
                                       FAKE, 1 << 30, S) == psa.PSA_ERR_ARG
    assert L.psa_route_thresh_prob(FAKE, FAKE, 1, 2, 16, 64, 0.5, 0, 0, FAKE, FAKE, 1 << 20, FAKE, None, FAKE, 16,
                                   S) == psa.PSA_ERR_CAPACITY
    # misaligned row maxima (routers' output, attention's input)
    odd = ctypes.c_void_p((1 << 20) + 2)
    assert L.psa_route_topk(FAKE, FAKE, 1, 2, 16, 64, 0.25, 0, FAKE, FAKE, 1 << 20, FAKE, odd, FAKE, 1 << 40, S) \
        == psa.PSA_ERR_ARG
    assert L.psa_attn(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 64, odd, 1, 2, 1024, 64, 64, 0, FAKE,
                      None, FAKE, ws, S) == psa.PSA_ERR_ARG
    assert L.psa_dense(FAKE, FAKE, FAKE, 1, 2, 1024, 64, 3, FAKE, None, FAKE, ws, S) == psa.PSA_ERR_ARG
    assert L.psa_read_status(None, None, S) == psa.PSA_ERR_ARG


def test_binding_names_match_c_entry_points():
    for name in ("psa_pool", "psa_route_topk", "psa_route_thresh", "psa_attn", "psa_dense",
                 "psa_workspace_size", "psa_route_capacity", "psa_read_status"):
        assert callable(getattr(psa, name))


def test_no_cpu_fallback_in_product_package():
    """The product package never imports the oracle."""
    pkg = os.path.join(ROOT, "block_sparse_attention_psa_b200")
    for dirpath, _, files in os.walk(pkg):
        for fn in files:
            if fn.endswith((".py", ".cu", ".cuh", ".h")):
                with open(os.path.join(dirpath, fn)) as f:
                    src = f.read()
                assert "oracle" not in re.sub(r"#.*|//.*", "", src).replace("oracle.", "ORACLE") or \
                    "import oracle" not in src, fn
                assert "import oracle" not in src and "from oracle" not in src, fn


def test_binding_signatures_match_the_header():
    """Every PSA_API prototype in include/psa.h against the ctypes signature
    the binding declares: same arity, and each parameter of the same kind
    (pointer, int, size_t, float)."""
    import re

    L = psa.lib()
    text = open(os.path.join(ROOT, "include", "psa.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    protos = re.findall(r"PSA_API\s+([\w\s\*]+?)\s*\b(psa_\w+)\s*\(([^;]*?)\)\s*;", text, flags=re.S)
    assert {name for _, name, _ in protos} == set(psa.EXPORTS)

    def kind(c_decl):
        c_decl = " ".join(c_decl.split())
        if "*" in c_decl:
            return "ptr"
        base = c_decl.replace("const ", "").split(" ")[0]
        return {"int": "int", "size_t": "size_t", "float": "float"}[base]

    ctype_kind = {ctypes.c_void_p: "ptr", ctypes.c_int: "int", ctypes.c_size_t: "size_t",
                  ctypes.c_float: "float"}
    for ret, name, params in protos:
        params = " ".join(params.split())
        c_params = [] if params in ("", "void") else [p.strip() for p in params.split(",")]
        fn = getattr(L, name)
        assert len(fn.argtypes) == len(c_params), name
        for c_decl, t in zip(c_params, fn.argtypes):
            want = kind(c_decl)
            got = "ptr" if t not in ctype_kind else ctype_kind[t]   # POINTER(...) types are pointers
            assert got == want, (name, c_decl, t)


def test_workspace_size_holds_the_documented_parts():
    """psa_workspace_size = pooled data O(B*H*M*d) + threshold masks + the
    first-order mode's per-query weights and partial statistics + the
    block-score matrices of as many heads as fit 256 MB (at least one head,
    4*M*Mp bytes, Mp = M rounded up to 128)."""
    def parts(B, H, M, d):
        bh = B * H
        Mp = -(-M // 128) * 128
        head = 4 * M * Mp
        heads = max(1, min(bh, (256 << 20) // head))
        # fixup lists (two), per-query log2 denominators, bf16 kbar / vsum,
        # threshold row counts, three-part splits of qbar and kbar
        pooled = 2 * bh * M * 4 + bh * M * 64 * 4 + 2 * bh * M * d * 2 + bh * M * 4 + 2 * 3 * bh * M * d * 2
        masks = bh * M * (-(-M // 32)) * 4
        # first-order mode: w per query, and one d x d partial per (head,
        # chunk of blocks), chunks sized for up to 256 SMs (2 CTAs each)
        want = min(M, max(1, -(-512 // bh)))
        per = -(-M // want)
        chunks = -(-M // per)
        hyd = bh * M * 64 * 4 + bh * chunks * d * d * 4
        # backward: two halves of partial pseudo-key gradients, one 128 x d
        # tile per (head, tile of 128 pooled keys, range of query blocks)
        items = bh * (-(-M // 128))
        want_b = min(M, max(1, -(-512 // items)))
        per_b = -(-M // want_b)
        bwd = 2 * items * (-(-M // per_b)) * 128 * d * 4
        return pooled + masks + hyd + bwd + heads * head

    for B, H, M, d in ((1, 12, 512, 128), (1, 8, 2048, 128), (1, 24, 1024, 64), (1, 2, 8192, 64),
                       (1, 1, 16384, 64), (2, 3, 37, 64)):
        got = psa.psa_workspace_size(B, H, M * 64, d)
        want = parts(B, H, M, d)
        # each region is rounded up to 256 bytes (header + 14 regions)
        assert want <= got <= want + 256 * 16, (B, H, M, d, got, want)
    # two heads of M = 8192 do not fit 256 MB together: one head's matrix is held
    one = psa.psa_workspace_size(1, 1, 8192 * 64, 64)
    two = psa.psa_workspace_size(1, 2, 8192 * 64, 64)
    assert two - one < 4 * 8192 * 8192
