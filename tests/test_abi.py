"""The C-ABI library loads and exports every entry point its headers declare (no GPU needed)."""
import ctypes
import glob
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s+\*?([A-Za-z_][A-Za-z0-9_]*)\s*\(",
                             text, flags=re.M):
            names.add(m.group(1))
    return names


def test_headers_declare_the_entry_points():
    want = {"sparse_prune_24", "sparse_compress_24", "tw_reorganize", "spgemm_24_f16", "spgemm_24_s8",
            "spgemm_tw_f16", "tw_query_sizes", "tw_workspace_size", "spg_version", "spg_status_string",
            "spg_check_device_error"}
    assert want <= _declared()


def test_library_exports_every_declared_symbol():
    import structured_sparse_gemm_02_b200 as spg
    L = spg.lib()
    for name in sorted(_declared()):
        assert hasattr(L, name), name
    assert set(spg.SIGNATURES) == _declared()


def test_host_only_calls():
    import structured_sparse_gemm_02_b200 as spg
    L = spg.lib()
    assert L.spg_version() == 10000
    assert L.spg_status_string(6) == b"SPG_ERR_TIMEOUT"
    sz = spg.SpgTwSizes()
    kpt = (ctypes.c_int32 * 6)(260, 290, 272, 118, 245, 187)
    assert L.tw_query_sizes(768, 768, 128, 77, kpt, ctypes.byref(sz)) == 0
    assert (sz.Nk, sz.T) == (691, 6)
    assert sz.offsetk_len == sum((k + 63) // 64 * 64 for k in (260, 290, 272, 118, 245, 187))
    assert sz.wc_elems == sz.offsetk_len * 128
    assert sz.reorg_ws_bytes >= 768 * 20
    assert L.tw_query_sizes(768, 768, 64, 77, kpt, ctypes.byref(sz)) == 2      # G must be 128
    assert L.tw_query_sizes(768, 768, 128, 768, kpt, ctypes.byref(sz)) == 1    # n_pruned < N
    one = (ctypes.c_int32 * 1)(768)
    assert L.tw_query_sizes(768, 768, 128, 767, one, ctypes.byref(sz)) == 0    # one kept column, all K rows
    assert (sz.Nk, sz.T, sz.offsetk_len) == (1, 1, 768)
    bad = (ctypes.c_int32 * 6)(260, 0, 272, 118, 245, 187)
    assert L.tw_query_sizes(768, 768, 128, 77, bad, ctypes.byref(sz)) == 1     # a tile keeping no row
    bad[1] = 769
    assert L.tw_query_sizes(768, 768, 128, 77, bad, ctypes.byref(sz)) == 1     # k_t > K
    assert L.tw_query_sizes(768, 760, 128, 77, kpt, ctypes.byref(sz)) == 2     # K % 64
    assert L.tw_query_sizes(768, 8256, 128, 77, kpt, ctypes.byref(sz)) == 2    # K above the reorganiser's limit
    assert L.tw_query_sizes(768, 768, 128, 77, None, ctypes.byref(sz)) == 1
    assert L.tw_workspace_size(4096, 768, spg.SPG_X_MK) == 4096 * 768 * 2
    # a ragged M: the transposed rows are padded to a multiple of 8 elements
    assert L.tw_workspace_size(15, 64, spg.SPG_X_MK) == (16 * 64 * 2 + 255) // 256 * 256
    assert L.tw_workspace_size(129, 768, spg.SPG_X_MK) == (136 * 768 * 2 + 255) // 256 * 256
    assert L.tw_workspace_size(4096, 768, spg.SPG_X_KM) == 0


def test_validation_rejects_before_touching_the_device():
    """Argument errors are reported on the host, before any device query or launch."""
    import structured_sparse_gemm_02_b200 as spg
    L = spg.lib()
    assert L.spgemm_24_f16(None, 256, None, None, None, None, 256, 64, 256, 256, 0, None) == 1
    assert L.spgemm_24_f16(16, 100, 16, 16, None, 16, 256, 64, 256, 256, 0, None) == 1   # ldx < K
    assert L.spgemm_24_f16(16, 256, 16, 16, None, 16, 256, 64, 256, 160, 0, None) == 2   # K % 64
    assert L.spgemm_24_f16(16, 256, 16, 16, None, 16, 256, 64, 256, 32, 0, None) == 2    # K < 64
    assert L.spgemm_24_f16(18, 256, 16, 16, None, 16, 256, 64, 256, 256, 0, None) == 3   # X misaligned
    assert L.spgemm_24_f16(16, 256, 16, 16, None, 16, 256, 64, 256, 256, 7, None) == 1   # dtype
    assert L.spgemm_24_s8(16, 256, 16, 16, None, None, 16, 256, 0, 64, 256, 256, None) == 1  # scale needed
    assert L.spgemm_24_s8(16, 256, 16, 16, None, None, 16, 256, 1, 64, 256, 192, None) == 2  # K % 128
    assert L.spgemm_24_s8(16, 256, 16, 16, None, None, 16, 256, 1, 64, 256, 64, None) == 2   # K < 128
    assert L.sparse_prune_24(16, 6, 16, 6, 2, 6, 0, None) == 2                               # K % 4
    assert L.sparse_compress_24(16, 12, 16, 16, 2, 12, 0, None) == 2                         # K % 8
    assert L.sparse_prune_24(16, 8, 16, 8, 0, 8, 0, None) == 0                               # empty: no-op
    # the host-buffer call: host pointers required for a non-empty batch, then the device layer's checks
    assert L.spgemm_24_f16_host(None, 256, 16, 16, None, 16, 256, 64, 256, 256, 0, 16, 16, 256, None) == 1
    assert L.spgemm_24_f16_host(16, 100, 16, 16, None, 16, 256, 64, 256, 256, 0, 16, 16, 256, None) == 1  # ldx_host
    assert L.spgemm_24_f16_host(16, 256, 16, 16, None, 16, 256, 64, 256, 160, 0, 16, 16, 256, None) == 2  # K % 64
    assert L.spgemm_24_f16_host(16, 256, 16, 16, None, 16, 256, 64, 256, 256, 0, 18, 16, 256, None) == 3  # X_dev
    assert L.spgemm_24_f16_host(None, 256, 16, 16, None, None, 256, 0, 256, 256, 0, None, None, 256, None) == 0
    # transposed outputs: the pitch of Y^T covers M, not N
    assert L.spgemm_24_f16_yt(16, 256, 16, 16, None, 16, 32, 64, 256, 256, 0, None) == 1  # ldyt < M
    assert L.spgemm_24_f16_yt(16, 256, 16, 16, None, 16, 68, 68, 256, 256, 0, None) == 3  # ldyt*2 % 16
    desc = spg.SpgTwDesc()
    desc.N, desc.K, desc.Nk, desc.G, desc.T, desc.offsetk_len = 768, 768, 691, 128, 6, 1536
    for f in ("offsetn", "tile_n0", "tile_kofs", "k_per_tile", "offsetk", "Wc"):
        setattr(desc, f, 256)
    assert L.spgemm_tw_f16_yt(16, 64, 1, ctypes.byref(desc), 16, 32, 64, None, 0, None) == 1  # ldyt < M
    assert L.spgemm_tw_f16_yt(16, 64, 1, ctypes.byref(desc), 18, 64, 64, None, 0, None) == 3  # Yt not 16-B aligned
    assert L.spgemm_tw_f16_yt(16, 64, 1, ctypes.byref(desc), 16, 68, 64, None, 0, None) == 3  # ldyt % 8


def test_tw_f32_validation_and_workspace_sizes():
    """The CUDA-core fp32 tile-wise entry points reject bad arguments on the host."""
    import structured_sparse_gemm_02_b200 as spg
    L = spg.lib()
    # [M, K] inputs are transposed at a pitch rounded up to 4 floats, in 256-byte units
    assert L.tw_workspace_size_f32(4095, 768, spg.SPG_X_MK) == (4096 * 768 * 4 + 255) // 256 * 256
    assert L.tw_workspace_size_f32(4096, 768, spg.SPG_X_KM) == 0
    assert L.tw_workspace_size_f32(0, 768, spg.SPG_X_MK) == 0
    desc = spg.SpgTwDesc()
    desc.N, desc.K, desc.Nk, desc.G, desc.T, desc.offsetk_len = 768, 768, 691, 128, 6, 1536
    for f in ("offsetn", "tile_n0", "tile_kofs", "k_per_tile", "offsetk", "Wc"):
        setattr(desc, f, 256)
    d = ctypes.byref(desc)
    X, W, Y, ws = 4096, 8192, 16384, 32768          # stand-in addresses, 16-byte aligned
    assert L.spgemm_tw_f32(None, 768, 0, d, W, Y, 768, 64, ws, 1 << 20, None) == 1        # no X
    assert L.spgemm_tw_f32(X, 768, 5, d, W, Y, 768, 64, ws, 1 << 20, None) == 1           # layout
    assert L.spgemm_tw_f32(X, 768, 0, d, W, Y, 700, 64, ws, 1 << 20, None) == 1           # ldy < N
    assert L.spgemm_tw_f32(X, 700, 0, d, W, Y, 768, 64, ws, 1 << 20, None) == 1           # ldx < K
    assert L.spgemm_tw_f32(X, 768, 0, d, W, Y, 768, 64, None, 0, None) == 1               # no workspace
    assert L.spgemm_tw_f32(X, 768, 0, d, W, Y, 768, 64, ws, 100, None) == 1               # workspace short
    assert L.spgemm_tw_f32(X + 4, 64, 1, d, W, Y, 768, 64, None, 0, None) == 3            # Xt rows not 16-B
    assert L.spgemm_tw_f32(X, 66, 1, d, W, Y, 768, 64, None, 0, None) == 3                # ldx % 4
    assert L.spgemm_tw_f32(X, 768, 0, d, W + 4, Y, 768, 64, ws, 1 << 20, None) == 3       # Wc32 alignment
    assert L.spgemm_tw_f32(X, 768, 0, d, W, Y + 2, 768, 64, ws, 1 << 20, None) == 3       # Y alignment
    assert L.tw_condense_f32(W, 700, d, W, None) == 1                                     # ldw < K
    assert L.tw_condense_f32(W, 768, d, W + 4, None) == 3                                 # Wc32 alignment
    desc.G = 64
    assert L.spgemm_tw_f32(X, 768, 0, d, W, Y, 768, 64, ws, 1 << 20, None) == 1           # G must be 128


def test_empty_batch_is_a_no_op():
    """M == 0 returns SPG_OK before anything touches the device (X, Y and the
    workspace may be NULL); the other arguments are still validated."""
    import structured_sparse_gemm_02_b200 as spg
    L = spg.lib()
    Wv, meta, sc = 4096, 8192, 12288                   # stand-in addresses, 16-byte aligned
    assert L.spgemm_24_f16(None, 256, Wv, meta, None, None, 256, 0, 256, 256, 0, None) == 0
    assert L.spgemm_24_f16_gelu(None, 256, Wv, meta, None, None, 256, 0, 256, 256, 1, None) == 0
    assert L.spgemm_24_f16_yt(None, 256, Wv, meta, None, None, 0, 0, 256, 256, 0, None) == 0
    assert L.spgemm_24_s8(None, 256, Wv, meta, sc, None, None, 256, 0, 0, 256, 256, None) == 0
    assert L.spgemm_24_s8_q(None, 256, Wv, meta, sc, None, ctypes.c_float(1.0), 0, None, 256, 0, 256, 256,
                            None) == 0
    # zero-size torch tensors report a row stride of 1 ([N, 0] outputs, [K, 0] inputs): not checked
    assert L.spgemm_24_f16_yt(None, 256, Wv, meta, None, None, 1, 0, 256, 256, 0, None) == 0
    assert L.spgemm_24_f16(None, 256, Wv, meta, None, None, 256, 0, 256, 160, 0, None) == 2   # K % 64
    assert L.spgemm_24_f16(None, 256, Wv, meta, None, None, 256, 0, 256, 192, 0, None) == 0   # K % 64 is enough
    assert L.spgemm_24_f16(None, 256, None, meta, None, None, 256, 0, 256, 256, 0, None) == 1  # no Wv
    assert L.spgemm_24_f16(None, 256, Wv, meta, None, None, 256, -1, 256, 256, 0, None) == 1  # M < 0
    assert L.spgemm_24_s8(None, 256, Wv, meta, None, None, None, 256, 0, 0, 256, 256, None) == 1  # scale
    desc = spg.SpgTwDesc()
    desc.N, desc.K, desc.Nk, desc.G, desc.T, desc.offsetk_len = 768, 768, 691, 128, 6, 1536
    for f in ("offsetn", "tile_n0", "tile_kofs", "k_per_tile", "offsetk", "Wc"):
        setattr(desc, f, 256)
    d = ctypes.byref(desc)
    assert L.tw_workspace_size(0, 768, spg.SPG_X_MK) == 0
    assert L.spgemm_tw_f16(None, 768, spg.SPG_X_MK, d, None, 768, 0, None, 0, None) == 0
    assert L.spgemm_tw_f16_yt(None, 1, spg.SPG_X_KM, d, None, 1, 0, None, 0, None) == 0
    assert L.spgemm_tw_f32(None, 1, spg.SPG_X_KM, d, Wv, None, 768, 0, None, 0, None) == 0
    assert L.spgemm_tw_f32(None, 768, spg.SPG_X_MK, d, Wv, None, 768, 0, None, 0, None) == 0
    assert L.spgemm_tw_f16(None, 768, spg.SPG_X_MK, d, None, 700, 0, None, 0, None) == 1      # ldy < N
    # the entry point without allocation keeps M >= 8 (its limits are its own)
    assert L.spgemm_tw_f16_noalloc(None, 768, d, None, 768, 0, None) == 1


def test_plain_c_program_uses_the_abi(tmp_path):
    """The header is valid C99 and every declared entry point links with C
    linkage: a C program takes the address of each one, links against the
    library and runs the host-only calls."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc not available")
    import structured_sparse_gemm_02_b200 as spg
    spg.lib()
    names = sorted(_declared())
    src = tmp_path / "use_abi.c"
    src.write_text(
        "#include <stdio.h>\n#include \"spgemm.h\"\n"
        "int main(void) {\n"
        "  void* fns[] = {" + ", ".join(f"(void*){n}" for n in names) + "};\n"
        "  int32_t kpt[6] = {260, 290, 272, 118, 245, 187};\n"
        "  spg_tw_sizes sz;\n"
        "  spg_status st = tw_query_sizes(768, 768, 128, 77, kpt, &sz);\n"
        "  for (unsigned i = 0; i < sizeof(fns) / sizeof(fns[0]); ++i) if (!fns[i]) return 2;\n"
        "  printf(\"%d %d %lld %d %s\\n\", spg_version(), (int)st, (long long)sz.Nk, sz.T,\n"
        "         spg_status_string(SPG_ERR_TIMEOUT));\n"
        "  return 0;\n}\n")
    libdir = os.path.dirname(spg.LIB_PATH)
    exe = tmp_path / "use_abi"
    p = subprocess.run([gcc, "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), str(src),
                        "-L", libdir, "-lspgemm", f"-Wl,-rpath,{libdir}", "-o", str(exe)],
                       capture_output=True, text=True)
    assert p.returncode == 0, p.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stderr
    assert r.stdout.split() == ["10000", "0", "691", "6", "SPG_ERR_TIMEOUT"]
