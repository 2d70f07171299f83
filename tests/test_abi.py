"""The C ABI without a GPU: libfm.so loads, exports every function that
include/fm.h declares, and its host-side calls (defaults, status text,
workspace sizing, argument checks that reject before any device work)
behave as the header states."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fm.h")
LIB = os.path.join(ROOT, "learned_kv_chunk_b200", "lib", "libfm.so")

if not os.path.exists(LIB):
    pytest.skip("libfm.so is not built (python -m learned_kv_chunk_b200.build)", allow_module_level=True)


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^[A-Za-z_][\w \*]*?\b(fm_\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    return ctypes.CDLL(LIB)


def test_header_declares_the_calls():
    names = declared_functions()
    for required in ["fm_create", "fm_destroy", "fm_query_prep", "fm_score", "fm_ensemble",
                     "fm_score_fused", "fm_select_topk", "fm_select_threshold",
                     "fm_topk_workspace_bytes", "fm_sync_status", "fm_strerror"]:
        assert required in names, required


def test_every_declared_function_is_exported(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", LIB], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\sT\s+(fm_\w+)$", out, flags=re.M))
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, missing
    for n in declared_functions():
        getattr(lib, n)  # resolvable through the dynamic loader too


def test_status_text(lib):
    lib.fm_strerror.restype = ctypes.c_char_p
    texts = [lib.fm_strerror(s).decode() for s in range(7)]
    assert texts[0] == "ok"
    assert len(set(texts)) == 7
    assert lib.fm_strerror(99).decode() == "unknown status"


def test_config_defaults(lib):
    from learned_kv_chunk_b200.fm import fm_config
    c = fm_config()
    lib.fm_config_default(ctypes.byref(c))
    assert (c.hidden, c.q_lora_rank, c.n_heads, c.head_dim, c.n_layers, c.rope_dim) == (4096, 1024, 64, 128, 3, 64)
    assert (c.rope_base, c.rope_factor, c.rope_orig_max_pos) == (160000.0, 16.0, 65536.0)
    assert (c.rope_beta_fast, c.rope_beta_slow) == (32.0, 1.0)
    assert abs(c.rms_eps - 1e-6) < 1e-12
    assert c.q_pieces in (2, 3) and c.max_batch >= 1
    assert c.cta_pairs == 0


def test_topk_workspace_sizing(lib):
    f = lib.fm_topk_workspace_bytes
    f.restype = ctypes.c_size_t
    f.argtypes = [ctypes.c_int, ctypes.c_int]
    assert f(0, 100) == 0 and f(1, 0) == 0
    a, b, c = f(1, 4096), f(2, 4096), f(1, 1 << 20)
    assert 0 < a < b and a < c
    assert a % 256 == 0 and c % 256 == 0
    # the no-allocation variant's limit covers the 64-row, 262144-chunk workload
    assert f(64, 262144) <= (4 << 20) < f(300, 262144)


def test_host_side_argument_rejection(lib):
    P, I = ctypes.c_void_p, ctypes.c_int
    lib.fm_select_topk.argtypes = [P, P, I, I, I, P, P, ctypes.c_size_t, P]
    lib.fm_select_topk_static.argtypes = [P, P, I, I, I, P, P]
    lib.fm_select_threshold.argtypes = [P, P, I, I, ctypes.c_float, P, P]
    lib.fm_ensemble.argtypes = [P, I, I, I, I, P, P]
    fake = ctypes.c_void_p(0x1000)  # never dereferenced: every call below fails its checks first
    INVALID, ALIGN, UNSUP = 1, 2, 3
    assert lib.fm_select_topk(None, None, 1, 10, 5, fake, fake, 1 << 20, None) == INVALID
    assert lib.fm_select_topk(fake, None, 1, 10, 0, fake, fake, 1 << 20, None) == INVALID
    assert lib.fm_select_topk(fake, None, 1, 10, 5, fake, fake, 0, None) == INVALID
    assert lib.fm_select_topk(ctypes.c_void_p(0x1001), None, 1, 10, 5, fake, fake, 1 << 20, None) == ALIGN
    assert lib.fm_select_topk_static(fake, None, 300, 262144, 5, fake, None) == UNSUP
    assert lib.fm_select_topk_static(fake, None, 0, 10, 5, fake, None) == INVALID
    assert lib.fm_select_threshold(None, None, 1, 10, 0.5, fake, None) == INVALID
    assert lib.fm_ensemble(fake, 5, 1, 10, 0, fake, None) == INVALID  # more layers than supported
    assert lib.fm_ensemble(fake, 3, 1, 10, 7, fake, None) == INVALID  # unknown mode
    S = ctypes.c_size_t
    lib.fm_topk_shard_begin.argtypes = [P, I, I, I, P, P, S, P]
    lib.fm_topk_shard_hist.argtypes = [P, I, I, I, P, P, S, P]
    lib.fm_topk_shard_pick.argtypes = [I, I, I, P, P, S, P]
    lib.fm_topk_shard_mask.argtypes = [P, I, I, P, I, P, P, S, P]
    assert lib.fm_topk_shard_begin(None, 1, 10, 0, fake, fake, 1 << 20, None) == INVALID  # k < 1
    assert lib.fm_topk_shard_begin(None, 1, 10, 5, ctypes.c_void_p(0x1004), fake, 1 << 20, None) == ALIGN
    assert lib.fm_topk_shard_hist(fake, 1, 10, 3, fake, fake, 1 << 20, None) == INVALID  # pass 3
    assert lib.fm_topk_shard_pick(1, 10, 0, fake, fake, 16, None) == INVALID  # workspace too small
    assert lib.fm_topk_shard_mask(fake, 1, 10, fake, -1, fake, fake, 1 << 20, None) == INVALID
    lib.fm_create.argtypes = [P, P, I, ctypes.POINTER(P)]
    out = P(0x1234)
    assert lib.fm_create(None, None, 0, ctypes.byref(out)) == INVALID
    assert out.value is None


def test_recall_argument_rejection(lib):
    """The recall calls refuse bad arguments on the host, before any CUDA
    call: null pointers, sizes below one, strides that cannot hold a row,
    misaligned index lists, a workspace that is too small."""
    P, I, I64, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
    lib.fm_compact_mask.argtypes = [P, I, I, I, P, P, P, S, P]
    lib.fm_gather_records.argtypes = [P, I64, I, I64, P, P, I, I, P, I64, P]
    fake = ctypes.c_void_p(0x1000)  # never dereferenced: every call below fails its checks first
    INVALID, ALIGN = 1, 2
    ws = int(lib.fm_compact_workspace_bytes(4, 1000))
    assert ws > 0
    assert lib.fm_compact_mask(None, 4, 1000, 64, fake, fake, fake, ws, None) == INVALID
    assert lib.fm_compact_mask(fake, 0, 1000, 64, fake, fake, fake, ws, None) == INVALID
    assert lib.fm_compact_mask(fake, 4, 1000, 0, fake, fake, fake, ws, None) == INVALID
    assert lib.fm_compact_mask(fake, 70000, 1000, 64, fake, fake, fake, ws, None) == INVALID  # B > 65535
    assert lib.fm_compact_mask(fake, 4, 1000, 64, ctypes.c_void_p(0x1002), fake, fake, ws, None) == ALIGN
    assert lib.fm_compact_mask(fake, 4, 1000, 64, fake, fake, ctypes.c_void_p(0x1008), ws, None) == ALIGN
    assert lib.fm_compact_mask(fake, 4, 1000, 64, fake, fake, fake, ws - 1, None) == INVALID
    assert lib.fm_gather_records(None, 1320, 10, 132, fake, fake, 4, 8, fake, 1056, None) == INVALID
    assert lib.fm_gather_records(fake, 1320, 10, 0, fake, fake, 4, 8, fake, 1056, None) == INVALID
    assert lib.fm_gather_records(fake, 1319, 10, 132, fake, fake, 4, 8, fake, 1056, None) == INVALID  # row stride
    assert lib.fm_gather_records(fake, 1320, 10, 132, fake, fake, 4, 8, fake, 1055, None) == INVALID  # dst stride
    assert lib.fm_gather_records(fake, 1320, 10, 132, ctypes.c_void_p(0x1001), fake, 4, 8, fake, 1056,
                                 None) == ALIGN


def test_header_is_plain_c(tmp_path):
    """include/fm.h is a C ABI: it compiles as strict C99 (and as C++), with
    every declared type usable from C."""
    import shutil
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "use_fm.c"
    src.write_text('#include "fm.h"\n'
                   "int main(void) {\n"
                   "  fm_config c; fm_config_default(&c);\n"
                   "  fm_layer_weights w; fm_level2_desc d; (void)w; (void)d;\n"
                   "  return (int)(fm_topk_workspace_bytes(1, 10) == 0) + (int)FM_TOPK_SHARD_BINS * 0;\n"
                   "}\n")
    r = subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-fsyntax-only",
                        "-I", os.path.dirname(HEADER), str(src)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr


def test_topk_fast_workspace_sizing(lib):
    """The candidate path's workspace adds, per row, a threshold, a count and a
    list of min(16384, max(256, N/16)) (key, index) pairs to the base workspace;
    the base one alone still fits the no-allocation scratch for 64 x 262144."""
    f, g = lib.fm_topk_workspace_bytes, lib.fm_topk_workspace_bytes_fast
    for fn in (f, g):
        fn.restype = ctypes.c_size_t
        fn.argtypes = [ctypes.c_int, ctypes.c_int]
    assert g(0, 10) == 0 and g(1, 0) == 0
    for B, N in [(1, 4096), (64, 262144), (8, 65536), (32, 131072), (3, 1 << 22)]:
        cap = min(16384, max(256, (N + 15) // 16))
        extra = g(B, N) - f(B, N)
        assert extra >= 2 * 4 * B * cap and extra <= 2 * 4 * B * cap + 4 * 256, (B, N, extra)
        assert g(B, N) % 256 == 0
    assert f(64, 262144) <= (4 << 20) < g(64, 262144)
