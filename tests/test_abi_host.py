"""The C-ABI library loads and exports what include/flarepp.h declares, and its
host-side argument checks answer before any CUDA call (no GPU needed)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", f) for f in sorted(os.listdir(os.path.join(ROOT, "include")))
           if f.endswith(".h")]


@pytest.fixture(scope="module")
def lib():
    from rank_latent_attention_mixer_b200 import build
    build.build()
    from rank_latent_attention_mixer_b200 import binding
    return binding


def declared_functions():
    names = []
    for h in HEADERS:
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names += re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*(flare[a-z0-9_]*)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_header_declares_entries():
    names = declared_functions()
    for required in ("flarepp_mixer_fwd", "flare_fwd", "flarepp_workspace_bytes", "flarepp_status_string"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib.lib, name), f"libflarepp.so does not export {name}"
    assert set(lib.EXPORTS) <= set(declared_functions())


def test_abi_version_and_status_strings(lib):
    assert lib.lib.flarepp_abi_version() == 5
    assert lib.bwd_launches(True) == 14 and lib.bwd_launches(False) == 9
    assert lib.bwd_launches(True, lib.PATH_TCGEN05) == 14 and lib.bwd_launches(False, lib.PATH_TCGEN05) == 9
    assert lib.launches_per_call(True) == 5 and lib.launches_per_call(False) == 3
    for code in range(6):
        assert lib.status_string(code) not in ("", "unknown status")
    assert lib.status_string(99) == "unknown status"


def _fwd(lib, ptrs, B=1, H=2, N=64, M=16, D=16, dtype=1):
    return lib.lib.flarepp_mixer_fwd(*ptrs, B, H, N, M, D, dtype, None)


FAKE = [0x10000, 0x20000, 0x30000, 0x40000, 0x50000, 0x60000, 0x70000]  # 16-byte aligned, never dereferenced


def test_null_pointers_rejected(lib):
    for i in (1, 4, 5, 6):        # q_fixed, k, v, y are always required
        p = list(FAKE)
        p[i] = None
        assert _fwd(lib, p) == 1
    p = list(FAKE)
    p[0] = None                   # q0 required when the gate is open
    assert _fwd(lib, p) == 1
    p[3] = None                   # k0 as well
    assert _fwd(lib, p) == 1


def test_bad_sizes_and_dtype(lib):
    assert _fwd(lib, FAKE, B=0) == 1
    assert _fwd(lib, FAKE, N=0) == 1
    assert _fwd(lib, FAKE, M=-3) == 1
    assert _fwd(lib, FAKE, dtype=7) == 1
    assert _fwd(lib, FAKE, D=48) == 2
    assert _fwd(lib, FAKE, D=256) == 2
    assert _fwd(lib, FAKE, M=5000) == 2
    assert _fwd(lib, FAKE, B=300, H=300) == 2


def test_misaligned_and_overlapping_rejected(lib):
    p = list(FAKE)
    p[4] = 0x20008                # k misaligned
    assert _fwd(lib, p) == 1
    p = list(FAKE)
    p[6] = p[5] + 16              # y overlaps v
    assert _fwd(lib, p) == 1
    p = list(FAKE)
    p[2] = 0x30002                # gate not 4-byte aligned
    assert _fwd(lib, p) == 1


def test_options_checked(lib):
    o = lib.Options(0.0, 9, 0, 0, None, None, None, 0, None)
    rc = lib.lib.flarepp_mixer_fwd_ex(*FAKE, 1, 2, 64, 16, 16, 1, ctypes.byref(o), None)
    assert rc == 1
    o = lib.Options(0.0, 0, 0, 5, None, None, None, 0, None)   # events promised, none given
    rc = lib.lib.flarepp_mixer_fwd_ex(*FAKE, 1, 2, 64, 16, 16, 1, ctypes.byref(o), None)
    assert rc == 1
    o = lib.Options(0.0, 0, 0, 0, None, None, 0x1000, 16, None)   # workspace too small
    rc = lib.lib.flarepp_mixer_fwd_ex(*FAKE, 1, 2, 64, 16, 16, 1, ctypes.byref(o), None)
    assert rc == 4
    o = lib.Options(0.0, 0, 0, 0, None, None, None, 0, None, 2)     # unknown token layout
    assert lib.lib.flarepp_mixer_fwd_ex(*FAKE, 1, 2, 64, 16, 16, 1, ctypes.byref(o), None) == 1
    assert lib.workspace_bytes(1, 2, 64, 16, 16, lib.BF16, layout="bnhd") == lib.workspace_bytes(1, 2, 64, 16, 16,
                                                                                                  lib.BF16)


def test_workspace_and_path_queries(lib):
    assert lib.workspace_bytes(1, 2, 1024, 16, 16, lib.F32) > 0
    assert lib.workspace_bytes(1, 2, 1024, 16, 48, lib.F32) == 0
    assert lib.selected_path(1, 2, 1024, 16, 16, lib.F32) == lib.PATH_SIMT
    assert lib.selected_path(1, 2, 1024, 16, 48, lib.F32) == 0
    # more forced chunks -> more partial triples -> more scratch
    a = lib.workspace_bytes(1, 8, 100000, 64, 32, lib.BF16, force_chunks=1)
    b = lib.workspace_bytes(1, 8, 100000, 64, 32, lib.BF16, force_chunks=16)
    assert 0 < a < b
    # 16-bit I/O plans the tcgen05 path for every supported D; fp32 the SIMT path
    assert lib.selected_path(1, 8, 100000, 64, 32, lib.F16) == lib.PATH_TCGEN05
    assert lib.selected_path(1, 8, 100000, 64, 128, lib.F16) == lib.PATH_TCGEN05
    assert lib.selected_path(1, 8, 100000, 64, 128, lib.BF16) == lib.PATH_TCGEN05
    assert lib.selected_path(1, 8, 100000, 64, 128, lib.F32) == lib.PATH_SIMT
    assert lib.workspace_bytes(1, 8, 100000, 64, 32, lib.F16) == lib.workspace_bytes(1, 8, 100000, 64, 32, lib.BF16)


def test_flare_entry_checks(lib):
    assert lib.lib.flare_fwd(None, FAKE[4], FAKE[5], FAKE[6], 1, 2, 64, 16, 16, 1, None) == 1
    assert lib.lib.flare_fwd(FAKE[1], FAKE[4], FAKE[5], FAKE[6], 1, 2, 64, 16, 40, 1, None) == 2


def test_token_sharded_entries_checked(lib):
    assert lib.cp_triple_bytes(1, 2, 16, 16) == 1 * 2 * 16 * 18 * 4
    assert lib.cp_latent_bytes(1, 2, 16, 16, lib.F32) == 2048
    assert lib.cp_latent_bytes(1, 2, 16, 16, lib.BF16) == 2048 + 1024
    assert lib.cp_triple_bytes(1, 2, 16, 48) == 0                       # D outside the supported set
    vp, i = ctypes.c_void_p, ctypes.c_int
    merge = lib.lib.flarepp_cp_merge
    merge.argtypes = [vp, i, vp, vp, vp, i, i, i, i, i, vp]
    assert merge(FAKE[4], 0, None, None, FAKE[6], 1, 2, 16, 16, 1, None) == 1     # no ranks
    assert merge(FAKE[4], 2, None, FAKE[2], FAKE[6], 1, 2, 16, 16, 1, None) == 1  # gate without q_fixed
    part = lib.lib.flarepp_cp_partials
    part.argtypes = [vp, i, vp, vp, vp, i, i, i, i, i, i, vp, vp]
    assert part(FAKE[1], 2, FAKE[4], FAKE[5], FAKE[6], 1, 2, 64, 16, 16, 1, None, None) == 1   # q_shared not 0/1
    assert part(FAKE[1], 1, FAKE[4], FAKE[5], None, 1, 2, 64, 16, 16, 1, None, None) == 1      # no triple
    dec = lib.lib.flarepp_cp_decode
    dec.argtypes = [vp, i, vp, vp, vp, i, i, i, i, i, i, vp, vp]
    assert dec(FAKE[1], 1, FAKE[3], FAKE[4], FAKE[4], 1, 2, 64, 16, 16, 1, None, None) == 1   # y aliases k


def _bwd(lib, ptrs, B=1, H=2, N=64, M=16, D=16, dtype=1, opts=None):
    return lib.lib.flarepp_mixer_bwd(*ptrs, B, H, N, M, D, dtype, opts, None)


# q0, q_fixed, gate, k0, k, v, dy | dq0, dq_fixed, dgate, dk0, dk, dv (16-byte aligned, never dereferenced)
BWD = [0x100000 * (i + 1) for i in range(13)]


def test_backward_entry_checks(lib):
    for i in (1, 4, 5, 6, 8, 11, 12):      # always required
        p = list(BWD)
        p[i] = None
        assert _bwd(lib, p) == 1, i
    for i in (0, 3, 7, 9, 10):             # required with the gate open
        p = list(BWD)
        p[i] = None
        assert _bwd(lib, p) == 1, i
    p = list(BWD)
    p[2] = None                            # closed gate: q0, k0, dq0, dgate, dk0 not needed, but no GPU here:
    for i in (0, 3, 7, 9, 10):             # the call gets past the checks and fails on the allocation
        p[i] = None
    assert _bwd(lib, p) in (3, 4)
    p = list(BWD)
    p[11] = p[4] + 32                      # dk overlaps k
    assert _bwd(lib, p) == 1
    p = list(BWD)
    p[12] = p[11]                          # dv aliases dk
    assert _bwd(lib, p) == 1
    p = list(BWD)
    p[6] = p[6] + 8                        # dy misaligned
    assert _bwd(lib, p) == 1
    assert _bwd(lib, BWD, D=48) == 2
    assert _bwd(lib, BWD, B=0) == 1
    o = lib.Options(0.0, 0, 0, 0, None, None, None, 0, None, 0, 2)   # norm_synthesis must be 0 or 1
    assert _bwd(lib, BWD, opts=ctypes.byref(o)) == 1
    # norm_synthesis: the workspace grows by the normalised copies of q0 and k0
    assert lib.bwd_workspace_bytes(1, 2, 1000, 64, 32, lib.BF16, norm_synthesis=True) > \
        lib.bwd_workspace_bytes(1, 2, 1000, 64, 32, lib.BF16)
    o = lib.Options(0.0, 0, 0, 0, None, None, 0x1000, 16, None)      # workspace too small
    assert _bwd(lib, BWD, opts=ctypes.byref(o)) == 4


def test_backward_workspace_query(lib):
    a = lib.bwd_workspace_bytes(1, 2, 1000, 64, 32, lib.BF16)
    assert a > lib.workspace_bytes(1, 2, 1000, 64, 32, lib.BF16)
    assert lib.bwd_workspace_bytes(1, 2, 1000, 64, 48, lib.BF16) == 0
    # SIMT: the fp32 buffer of the decode's share of dk dominates (B*H*N*D*4 bytes);
    # tensor cores: per-token statistics only (the token sides are fused)
    big = lib.bwd_workspace_bytes(1, 8, 1 << 20, 512, 64, lib.BF16, path=lib.PATH_SIMT)
    assert big > 8 * (1 << 20) * 64 * 4
    assert lib.bwd_workspace_bytes(1, 8, 1 << 20, 512, 64, lib.BF16) < 8 * (1 << 20) * 64 * 2
    assert lib.bwd_workspace_bytes(1, 2, 1000, 64, 32, lib.BF16, force_chunks=1) < a


def test_training_context_entries_checked(lib):
    assert lib.train_context_bytes(1, 2, 1000, 64, 32, lib.BF16) > 0
    assert lib.train_context_bytes(1, 2, 1000, 64, 48, lib.BF16) == 0
    # the per-token log-sum-exps dominate at many tokens: B*H*N*8 bytes
    assert lib.train_context_bytes(1, 8, 1 << 20, 512, 64, lib.BF16) >= 8 * (1 << 20) * 8
    fwd = lib.lib.flarepp_mixer_fwd_train
    args = FAKE + [1, 2, 64, 16, 16, 1, None]
    assert fwd(*args, None, 1 << 20, None) == 1                  # no context
    assert fwd(*args, 0x900010, 1 << 20, None) == 1              # misaligned context
    assert fwd(*args, 0x900000, 16, None) == 4                   # context too small
    bwd = lib.lib.flarepp_mixer_bwd_ctx
    p = BWD[:6] + [0xe00000] + BWD[6:]                           # ... y, dy, grads
    assert bwd(*p, 1, 2, 64, 16, 16, 1, None, None, 1 << 20, None) == 1     # no context
    p2 = list(p)
    p2[6] = None                                                  # no y
    assert bwd(*p2, 1, 2, 64, 16, 16, 1, None, 0x900000, 1 << 20, None) == 1


def test_sharded_backward_entries_checked(lib):
    lay = lib.cp_bwd_layout(1, 2, 64, 16, 16, lib.BF16)
    assert lay.bytes > 0
    latd = 1 * 2 * 16 * 16 * 4
    assert list(lay.reduce_bytes) == [2 * latd, latd, latd]
    assert lay.reduce_offset[0] % 256 == 0 and lay.reduce_offset[1] >= lay.reduce_offset[0] + 2 * latd
    with pytest.raises(lib.FlareppError):
        lib.cp_bwd_layout(1, 2, 64, 16, 48, lib.BF16)
    fn = lib.lib.flarepp_cp_bwd_stage
    vp, i = ctypes.c_void_p, ctypes.c_int
    fn.argtypes = [i] + [vp] * 19 + [i] * 6 + [vp, vp]
    ptrs = [0x100000 * (j + 1) for j in range(19)]
    assert fn(0, *ptrs, 1, 2, 64, 16, 16, 1, None, None) == 1        # stage outside 1..4
    assert fn(5, *ptrs, 1, 2, 64, 16, 16, 1, None, None) == 1
    p = list(ptrs)
    p[18] = 0x100010                                                  # state misaligned
    assert fn(1, *p, 1, 2, 64, 16, 16, 1, None, None) == 1
    p = list(ptrs)
    p[4] = None                                                       # no z state
    assert fn(1, *p, 1, 2, 64, 16, 16, 1, None, None) == 1


def test_debug_and_workspace_entries_checked(lib):
    L = lib.lib
    # flarepp_mixer_fwd_debug: argument checks before any CUDA call
    assert L.flarepp_mixer_fwd_debug(*FAKE, 1, 2, 64, 16, 16, 1, None, None, -1, None) == 1   # force_chunks < 0
    ptrs = list(FAKE)
    ptrs[6] = None                                                                              # y NULL
    assert L.flarepp_mixer_fwd_debug(*ptrs, 1, 2, 64, 16, 16, 1, None, None, 0, None) == 1
    assert L.flarepp_mixer_fwd_debug(*FAKE, 1, 2, 64, 16, 48, 1, None, None, 0, None) == 2    # D = 48
    assert L.flarepp_mixer_fwd_debug(*FAKE, 1, 2, 64, 16, 16, 1, 0x10008, None, 0, None) == 1  # q_out misaligned
    # flarepp_set_workspace: a misaligned buffer is refused before any CUDA call
    assert L.flarepp_set_workspace(0x10010, 1 << 20) == 1


def test_noalloc_checks_pointers_before_cuda(lib):
    fn = lib.lib.flarepp_mixer_fwd_noalloc
    vp, i = ctypes.c_void_p, ctypes.c_int
    fn.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, vp]
    ptrs = list(FAKE)
    ptrs[6] = None                                  # y NULL
    assert fn(*ptrs, 1, 2, 64, 16, 16, 1, None) == 1
    ptrs = list(FAKE)
    ptrs[6] = FAKE[4]                               # y overlaps k
    assert fn(*ptrs, 1, 2, 64, 16, 16, 1, None) == 1
    ptrs = list(FAKE)
    ptrs[6] = 0x70008                               # y misaligned
    assert fn(*ptrs, 1, 2, 64, 16, 16, 1, None) == 1
