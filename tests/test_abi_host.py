"""Host-side checks of the C-ABI library (no GPU needed).

The library must load on a machine without a GPU, export every function that
include/fi_nvfp4.h declares, resolve tactics from a given SM count without touching CUDA,
and reject bad arguments before any CUDA call.
"""
import ctypes
import os
import re

import pytest

import bf16_activations_nvfp4_b200 as fi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fi_nvfp4.h")
B200_SMS = 148


def _declared_functions():
    text = open(HEADER).read()
    return re.findall(r"^FI_API\s+[\w\s\*]+?\b(fi_\w+)\s*\(", text, flags=re.M)


def test_library_exports_every_declared_symbol():
    names = _declared_functions()
    assert len(names) >= 11
    lib = fi.library()
    for name in names:
        assert hasattr(lib, name), name


def test_version():
    assert fi.version() >= 100


def test_tactic_encoding_matches_header_macros():
    t = fi.make_tactic(fi.KIND_MMA, 37, 3, 2)
    assert t == (1 << 24) | (37 << 12) | (3 << 8) | 2
    assert fi.tactic_fields(t) == {"kind": 1, "splits": 37, "ctas_per_sm": 3, "variant": 2}


@pytest.mark.parametrize("n,k", [(2048, 7168), (4096, 4096), (4096, 14336), (14336, 4096), (10304, 2688),
                                 (512, 2048), (512, 4096), (1024, 2048), (1024, 4096), (2048, 2048),
                                 (2048, 4096), (152064, 5120)])
def test_default_gemv_tactic_resolves_for_decode_shapes(n, k):
    info = fi.resolve_tactic(1, n, k, fi.TACTIC_DEFAULT, B200_SMS)
    tuned = {(e[0], e[1]): e[5] for e in _tuned_entries() if e[2] == 1 and e[4] == B200_SMS}
    assert info["kind"] == fi.KIND_GEMV
    assert 1 <= info["splits"] <= k // 32
    # one persistent wave: the grid never asks for more CTAs than the SMs hold
    assert info["grid_x"] * info["grid_y"] <= B200_SMS * info["ctas_per_sm"]
    # the default runs the per-warp async-copy pipeline (its lean form where k % 2048 == 0): one
    # CTA of up to 16 warps per SM, or two of up to 8 warps within half an SM each; weights of at
    # most 12 MB take the overlapped variant (one half-SM CTA per SM). Fewer warps only where the row groups would otherwise
    # leave SMs idle, and then the grid spans every SM of the split's share
    pipe = info["variant"] >> 4
    small = n * (k // 2 + k // 16) <= 12 << 20
    if (n, k) in tuned:  # the generated table decides: its pick is the default
        assert fi.default_tactic(1, n, k, B200_SMS) == tuned[(n, k)]
    else:
        assert pipe == (3 if small else (4 if k % 256 else (5 if k % 2048 == 0 else 1)))
    warps = info["threads"] // 32
    wide = 16
    if info["ctas_per_sm"] == 1:
        assert 4 <= warps <= wide and 0 < info["smem_bytes"] <= 227 * 1024 - 1024
    else:
        assert 4 <= warps <= wide // 2 and 0 < info["smem_bytes"] <= 228 * 1024 // 2 - 1024
    full = wide if info["ctas_per_sm"] == 1 else wide // 2
    if warps < full:
        share = B200_SMS * (1 if pipe == 3 else info["ctas_per_sm"]) // info["splits"]
        assert info["grid_x"] >= 0.95 * share or warps == 4, info  # whole groups per warp round the grid
    assert info["workspace_bytes"] == (info["splits"] * n * 4 if info["splits"] > 1 else 0)


def test_device_sized_split_is_m_independent():
    """The device-sized tactic (splits=0) resolves to the same S for every m the GEMV takes,
    and gives every SM a CTA unless the k range cannot be divided further."""
    for n, k in [(512, 2048), (1024, 4096), (4096, 14336), (14336, 4096), (2048, 7168), (10304, 2688)]:
        for R in (0, 1):
            t = fi.make_tactic(fi.KIND_GEMV, 0, 0, R)
            got = {fi.resolve_tactic(m, n, k, t, B200_SMS)["splits"] for m in (1, 2, 3, 8, 16, 32)}
            assert len(got) == 1, (n, k, R, got)
            info = fi.resolve_tactic(1, n, k, t, B200_SMS)
            assert info["grid_x"] * info["grid_y"] >= min(B200_SMS, info["grid_x"] * info["grid_y"])


def test_default_table_is_constant_within_m_buckets():
    """The generated table's buckets of m ({1}, {2}, {3, 4}, {5..32}, {33..256}) for the shapes
    it lists; the built-in rules' ({1}, {2..4}, {5..256}) for the others (3000 x 5120)."""
    tuned = ([1], [2], [3, 4], [5, 8, 16, 17, 32], [33, 64, 100, 256])
    builtin = ([1], [2, 3, 4], [5, 8, 16, 17, 32, 33, 64, 100, 256])
    for (n, k), buckets in [((4096, 14336), tuned), ((14336, 4096), tuned), ((512, 2048), tuned),
                            ((3000, 5120), builtin)]:
        for bucket in buckets:
            ts = {fi.default_tactic(m, n, k, B200_SMS) for m in bucket}
            assert len(ts) == 1, (n, k, bucket, ts)


def test_default_m1_serving_shapes_need_no_second_kernel():
    for n, k in [(2048, 7168), (4096, 4096), (4096, 14336), (14336, 4096), (10304, 2688), (152064, 5120)]:
        info = fi.resolve_tactic(1, n, k, fi.default_tactic(1, n, k, B200_SMS), B200_SMS)
        assert info["splits"] == 1 and info["workspace_bytes"] == 0, (n, k, info)


def test_explicit_splits_are_kept():
    for S in (1, 2, 4, 8):
        info = fi.resolve_tactic(1, 4096, 4096, fi.make_tactic(fi.KIND_GEMV, S, 0, 2), B200_SMS)
        assert info["splits"] == S and info["variant"] & 0xF == 2
    info = fi.resolve_tactic(1, 4096, 4096, fi.make_tactic(fi.KIND_GEMV, 2, 2, 1), B200_SMS)
    assert (info["splits"], info["ctas_per_sm"], info["variant"] & 0xF) == (2, 2, 1)
    ring = fi.resolve_tactic(1, 4096, 4096, fi.make_tactic(fi.KIND_GEMV, 2, 1, 0x21), B200_SMS)
    assert (ring["variant"], ring["threads"]) == (0x21, 17 * 32)


def test_list_tactics_unique_and_valid():
    ts = fi.list_tactics(1, 4096, 14336, B200_SMS)
    assert len(ts) == len(set(ts)) and len(ts) >= 6
    for t in ts:
        fi.resolve_tactic(1, 4096, 14336, t, B200_SMS)


def test_list_tactics_offers_the_mma_split_menu():
    """The MMA appears with splits 1, 2, 4, 8 and device-sized, one entry per distinct launch.
    Above m = 32 only MMA codes are listed; where k is not a multiple of 64, only GEMV codes."""
    ts = fi.list_tactics(64, 4096, 4096, B200_SMS)
    mma = [fi.resolve_tactic(64, 4096, 4096, t, B200_SMS) for t in ts if fi.tactic_fields(t)["kind"] == fi.KIND_MMA]
    assert {i["splits"] for i in mma} >= {1, 2, 4, 8}
    assert len({i["splits"] for i in mma}) == len(mma)
    assert all(fi.tactic_fields(t)["kind"] == fi.KIND_MMA for t in ts)  # m = 64 > the GEMV's 32
    assert all(fi.tactic_fields(t)["kind"] == fi.KIND_GEMV for t in fi.list_tactics(4, 1000, 1056, B200_SMS))


def test_workspace_bytes():
    t = fi.make_tactic(fi.KIND_GEMV, 4, 0, 1)
    assert fi.workspace_bytes(3, 1000, 4096, t, B200_SMS) == 4 * 3 * 1000 * 4
    assert fi.workspace_bytes(3, 1000, 4096, fi.make_tactic(fi.KIND_GEMV, 1, 0, 1), B200_SMS) == 0


@pytest.mark.parametrize("m,n,k,tactic,status", [
    (1, 64, 48, -1, -2),                                  # k % 32 != 0
    (33, 64, 64, fi.make_tactic(0, 1, 0, 1), -2),         # GEMV beyond m = 32
    (1, 64, 64, fi.make_tactic(0, 1, 0, 9), -1),          # rows per stage 9
    (1, 64, 64, fi.make_tactic(0, 1, 0, 3), -1),          # rows per stage not a power of two
    (1, 64, 64, fi.make_tactic(0, 3, 0, 1), -1),          # splits > k/32
    (1, 64, 64, fi.make_tactic(7, 1, 0, 1), -1),          # unknown kind
    (1, 64, 64, 1 << 30, -1),                             # out-of-range code
    (-1, 64, 64, -1, -1),                                 # negative size
    (32, 64, 14336, fi.make_tactic(0, 1, 0, 1), -2),      # A slice does not fit shared memory
    (32, 64, 4096, fi.make_tactic(0, 1, 0, 4), -1),       # one row per stage above m = 8
    (5, 64, 4096, fi.make_tactic(0, 1, 0, 4), -1),        # two rows per stage above m = 4
    (1, 64, 4096, fi.make_tactic(0, 1, 0, 0x62), -1),     # pipeline 6
    (1, 64, 2688, fi.make_tactic(0, 1, 0, 0x52), -2),     # the lean pipeline needs k % 256 == 0
    (1, 64, 4096, fi.make_tactic(0, 3, 0, 0x52), -2),     # ... and splits of whole 64-chunk items
    (2, 64, 4096, fi.make_tactic(0, 1, 0, 0x52), -2),     # the lean pipeline takes m = 1 only
    (1, 64, 4096, fi.make_tactic(0, 1, 0, 0x58), -1),     # lean pipeline: 1, 2 or 4 rows per item
    (1, 64, 4096, fi.make_tactic(0, 1, 0, 0x19), -1),     # rows 9 on the stream pipeline
    (1, 8, 65536, fi.make_tactic(0, 1, 0, 0x22), -2),     # ring: two 36 KB rows per stage do not fit twice
    (1, 8, 65536, fi.make_tactic(0, 1, 2, 0x11), -2),     # stream, half-SM CTAs: 128 KB of activations
])
def test_resolve_rejects(m, n, k, tactic, status):
    with pytest.raises(fi.FiError) as e:
        fi.resolve_tactic(m, n, k, tactic, B200_SMS)
    assert e.value.status == status
    assert fi.last_error()


def _call_mm(A, Wq, Ws, g, out, m, n, k, tactic=-1):
    lib = fi.library()
    return lib.fi_mm_bf16_fp4(A, Wq, Ws, g, out, m, n, k, tactic, None)


def test_mm_argument_checks_precede_cuda():
    lib = fi.library()
    # empty problems are no-ops
    assert _call_mm(None, None, None, None, None, 0, 64, 64) == 0
    assert _call_mm(None, None, None, None, None, 4, 0, 64) == 0
    # shape and pointer errors
    assert _call_mm(16, 16, 16, 16, 16, 1, 64, 40) == -2
    assert _call_mm(None, 16, 16, 16, 16, 1, 64, 64) == -1
    assert "null" in fi.last_error()
    assert _call_mm(0x1008, 0x2000, 0x3000, 0x4000, 0x5000, 1, 64, 64) == -1  # A misaligned
    assert "aligned" in fi.last_error()
    assert _call_mm(0x1000, 0x2000, 0x3008, 0x4000, 0x5000, 1, 64, 64) == -1  # Wscale not 16-byte aligned
    assert lib.fi_mm_bf16_fp4_ex(None, None, None, None, None, 0, 1, 32, -1, None, 0, None) == 0


def test_pack_and_reduce_argument_checks():
    lib = fi.library()
    assert lib.fi_nvfp4_pack_weights(0x1000, 4, 24, 0x2000, 0x3000, 0x4000, None) == -2
    assert lib.fi_nvfp4_pack_weights(0x1000, 4, 32, 0x2000, 0x3000, None, None) == -1
    assert lib.fi_nvfp4_pack_weights(0x1004, 4, 32, 0x2000, 0x3000, 0x4000, None) == -1
    assert lib.fi_nvfp4_pack_weights(0x1000, 4, 32, 0x2000, 0x3008, 0x4000, None) == -1
    assert lib.fi_splitk_reduce(0x1000, 0, 1, 1, 0x2000, 0x3000, None) == -1
    assert lib.fi_splitk_reduce(0x1000, 4096, 1, 1, 0x2000, 0x3000, None) == -1
    assert lib.fi_splitk_reduce(None, 2, 0, 5, None, None, None) == 0
    assert lib.fi_splitk_reduce(0x1008, 2, 1, 5, 0x2000, 0x3000, None) == -1


def test_set_workspace_rejects_bad_arguments():
    lib = fi.library()
    assert lib.fi_set_workspace(0x1000, 0) == -1
    assert lib.fi_set_workspace(None, 64) == -1
    assert lib.fi_set_workspace(0x1010, 4096) == -1


def test_debug_hooks_validate_arguments():
    with pytest.raises(fi.FiError):
        fi.debug_set(99, 1)
    with pytest.raises(fi.FiError):
        fi.debug_set(fi.DEBUG_WAIT_TIMEOUT_NS, 0)
    with pytest.raises(fi.FiError):
        fi.debug_set(fi.DEBUG_STALL_PRODUCER, -1)
    fi.debug_set(fi.DEBUG_STALL_PRODUCER, 0)
    fi.debug_set(fi.DEBUG_WAIT_TIMEOUT_NS, 1_000_000_000)
    assert fi.library().fi_get_device_error(None) == -1


def test_mma_tactic_resolution():
    t = fi.make_tactic(fi.KIND_MMA, 1, 0, 0)
    info = fi.resolve_tactic(256, 152064, 5120, t, B200_SMS)
    assert info["kind"] == fi.KIND_MMA and info["splits"] == 1
    assert info["grid_x"] == 152064 // 256 and info["threads"] == 24 * 32
    assert 0 < info["smem_bytes"] <= 227 * 1024
    # m = 256 (above the tensor-memory operand's 128 rows): the prepass conversion, whose
    # workspace is the f16 activations [256, k] then 256 fp32 (row, split) scales
    assert info["variant"] == 1
    assert info["workspace_bytes"] == 256 * 5120 * 2 + 256 * 4
    prepass = fi.make_tactic(fi.KIND_MMA, 1, 0, 1)
    assert fi.resolve_tactic(33, 100, 64, prepass, B200_SMS)["workspace_bytes"] == 48 * 64 * 2 + 48 * 4
    # resident activations (variant 2, converted in the kernel): no activation copy in the
    # workspace; the automatic variant takes them for m <= 8 (here one step)
    res = fi.resolve_tactic(33, 100, 64, fi.make_tactic(fi.KIND_MMA, 1, 0, 2), B200_SMS)
    assert (res["variant"], res["workspace_bytes"]) == (2, 0)
    assert fi.resolve_tactic(33, 100, 64, t, B200_SMS)["variant"] == 1
    res_t = fi.make_tactic(fi.KIND_MMA, 1, 0, 2)
    assert fi.resolve_tactic(8, 100, 64, t, B200_SMS) == fi.resolve_tactic(8, 100, 64, res_t, B200_SMS)
    assert fi.resolve_tactic(8, 100, 64, res_t, B200_SMS)["variant"] == 2
    assert fi.resolve_tactic(9, 100, 64, t, B200_SMS)["variant"] == 1
    # the built-in rules take the GEMV up to m = 4 and the MMA (device-sized split) above (a shape
    # the generated table does not list); the table's picks for 4096 x 4096 agree on the kind
    assert fi.resolve_tactic(5, 4096, 4096, fi.TACTIC_DEFAULT, B200_SMS)["kind"] == fi.KIND_MMA
    assert fi.resolve_tactic(4, 4096, 4096, fi.TACTIC_DEFAULT, B200_SMS)["kind"] == fi.KIND_GEMV
    assert fi.resolve_tactic(5, 4096, 12288, fi.TACTIC_DEFAULT, B200_SMS)["kind"] == fi.KIND_MMA
    assert fi.resolve_tactic(4, 4096, 12288, fi.TACTIC_DEFAULT, B200_SMS)["kind"] == fi.KIND_GEMV
    assert fi.resolve_tactic(32, 4096, 12288, fi.TACTIC_DEFAULT, B200_SMS)["splits"] == \
        fi.resolve_tactic(32, 4096, 12288, fi.make_tactic(fi.KIND_MMA, 0, 0, 0), B200_SMS)["splits"]
    assert t in fi.list_tactics(64, 4096, 4096, B200_SMS)


@pytest.mark.parametrize("m,n,k,tactic,status", [
    (257, 64, 64, fi.make_tactic(1, 1, 0, 0), -2),   # m beyond 256
    (64, 64, 96, fi.make_tactic(1, 1, 0, 0), -2),    # k not a multiple of 64
    (64, 64, 64, fi.make_tactic(1, 2, 0, 0), -1),    # no split-K on the MMA path
    (64, 64, 64, fi.make_tactic(1, 1, 0, 3), -1),    # variants 0 (automatic), 1 (prepass), 2 (resident)
    (129, 64, 64, fi.make_tactic(1, 1, 0, 2), -2),   # resident activations need m <= 128
    (16, 64, 64 * 97, fi.make_tactic(1, 1, 0, 2), -2),  # 97 steps x 16 rows x 128 B exceed shared memory
])
def test_mma_resolve_rejects(m, n, k, tactic, status):
    with pytest.raises(fi.FiError) as e:
        fi.resolve_tactic(m, n, k, tactic, B200_SMS)
    assert e.value.status == status


def test_mma_device_sized_split_follows_the_wave_step_model():
    """The MMA path's device-sized split (S = 0): one CTA per SM, so the choice is the S with the
    fewest waves of 64-k steps (per-CTA start and epilogue, the reduce and the partials
    counted). Small n needs a split, the lm_head-like shape does not."""
    mma = fi.make_tactic(fi.KIND_MMA, 0, 0, 0)
    cases = {(32, 4096, 14336): 9, (8, 4096, 14336): 9, (64, 152064, 5120): 1, (256, 152064, 5120): 1}
    for (m, n, k), S in cases.items():
        info = fi.resolve_tactic(m, n, k, mma, B200_SMS)
        assert info["splits"] == S and info["grid_y"] == S, (m, n, k, info)
        assert info["grid_x"] == -(-n // 256)
        if S > 1 and info["variant"] == 1:  # f16 activations, their scales, then the partials
            assert info["workspace_bytes"] >= S * m * n * 4 + 2 * 16 * k
        elif S > 1:  # resident activations: the partials only
            assert info["workspace_bytes"] == S * m * n * 4
    # explicit splits are kept, up to k / 64 steps
    assert fi.resolve_tactic(64, 4096, 4096, fi.make_tactic(fi.KIND_MMA, 3, 0, 0), B200_SMS)["splits"] == 3
    with pytest.raises(fi.FiError):
        fi.resolve_tactic(64, 4096, 128, fi.make_tactic(fi.KIND_MMA, 3, 0, 0), B200_SMS)


@pytest.mark.parametrize("n,k", [(4096, 14336), (14336, 4096), (2048, 7168), (4096, 4096), (152064, 5120),
                                 (512, 2048), (1000, 2688 + 64), (129, 1088)])
def test_mma_device_sized_split_does_not_depend_on_m(n, k):
    """A row's bits depend on the kind and the resolved S; the device-sized MMA split must
    therefore resolve to one S for every m (1..256), so that the code is batch-invariant."""
    mma = fi.make_tactic(fi.KIND_MMA, 0, 0, 0)
    splits = {fi.resolve_tactic(m, n, k, mma, B200_SMS)["splits"] for m in (1, 2, 5, 8, 16, 17, 32, 64, 100, 256)}
    assert len(splits) == 1, (n, k, splits)


def test_register_pipeline_geometry():
    """Pipeline 4: shared memory holds only the staged activations, 1 or 2 rows per warp, and
    the grid spreads over the SMs like the stream pipeline's."""
    for n, k in [(10304, 2688), (4096, 14336), (512, 2048)]:
        info = fi.resolve_tactic(1, n, k, fi.make_tactic(fi.KIND_GEMV, 1, 2, 0x40), B200_SMS)
        assert info["variant"] >> 4 == 4 and info["variant"] & 0xF == 2
        chunks = k // 32
        assert info["smem_bytes"] == -(-((chunks + 31) // 32 * 2048) // 128) * 128 + -(-(chunks * 8) // 128) * 128
        assert info["grid_x"] <= 2 * B200_SMS and info["threads"] % 32 == 0
    with pytest.raises(fi.FiError):
        fi.resolve_tactic(1, 4096, 4096, fi.make_tactic(fi.KIND_GEMV, 1, 0, 0x44), B200_SMS)  # 4 rows would spill


def _lean_fits(k, S):
    """The lean pipeline takes splits of whole 32-chunk iterations: k % 256 == 0, (k / 32) % (32 S) == 0."""
    return k % 256 == 0 and (k // 32) % (32 * S) == 0


def test_automatic_pipeline_for_split_calls_at_m1():
    """At m = 1 the automatic pipeline is the lean stream pipeline where its whole items fit the
    split; otherwise, with a K split, the register pipeline (two CTAs per SM) where k % 256 != 0
    and four rows per stream item elsewhere; S itself is unchanged, and m > 1 keeps the stream
    pipeline's own row choice."""
    for n, k in [(4096, 14336), (2048, 7168), (4096, 4096), (10304, 2688)]:
        for S in (2, 4, 8):
            info = fi.resolve_tactic(1, n, k, fi.make_tactic(fi.KIND_GEMV, S, 0, 0), B200_SMS)
            assert info["splits"] == S
            if _lean_fits(k, S):
                assert info["variant"] >> 4 == 5
            elif k % 256:
                assert (info["variant"] >> 4, info["ctas_per_sm"]) == (4, 2)
            else:
                assert info["variant"] == 0x14
        # S = 1: the lean pipeline where it fits, else the stream pipeline; the device-sized split
        # resolves to the same S at every m
        v1 = fi.resolve_tactic(1, n, k, fi.make_tactic(fi.KIND_GEMV, 1, 0, 0), B200_SMS)["variant"] >> 4
        assert v1 == (5 if _lean_fits(k, 1) else 1)
        s1 = fi.resolve_tactic(1, n, k, fi.make_tactic(fi.KIND_GEMV, 0, 0, 0), B200_SMS)["splits"]
        s4 = fi.resolve_tactic(4, n, k, fi.make_tactic(fi.KIND_GEMV, 0, 0, 0), B200_SMS)["splits"]
        assert s1 == s4
    # where those row groups would leave SMs with fewer than 4 warps, the stream pipeline keeps
    # its own row choice (n = 280: 70 four-row groups per split, 560 warps over 8 splits; S = 8
    # has no whole lean iterations at k = 4096)
    info = fi.resolve_tactic(1, 280, 4096, fi.make_tactic(fi.KIND_GEMV, 8, 0, 0), B200_SMS)
    assert info["variant"] >> 4 == 1 and info["variant"] & 15 != 4
    assert fi.resolve_tactic(1, 129, 2688, fi.make_tactic(fi.KIND_GEMV, 2, 0, 0), B200_SMS)["variant"] >> 4 == 1
    # explicit rows or pipeline are taken as given
    assert fi.resolve_tactic(1, 4096, 14336, fi.make_tactic(fi.KIND_GEMV, 2, 0, 0x12), B200_SMS)["variant"] == 0x12
    assert fi.resolve_tactic(1, 4096, 14336, fi.make_tactic(fi.KIND_GEMV, 2, 0, 0x01), B200_SMS)["variant"] & 15 == 1
    assert fi.resolve_tactic(2, 4096, 14336, fi.make_tactic(fi.KIND_GEMV, 2, 0, 0), B200_SMS)["variant"] >> 4 == 1


class _OnDevice:
    """Shape and device stand-in for a tensor on another GPU (no GPU needed)."""

    def __init__(self, t, index):
        self.shape, self._index = t.shape, index
        self.device = f"cuda:{index}"

    def get_device(self):
        return self._index


def test_binding_checks_shapes_and_devices_before_any_launch():
    """The Python binding refuses operands the kernels would read or write out of bounds:
    `out` must be [m, n], Wscale [n, k/16], gscale one element, and every operand on A's
    device; pack_weights' `out` buffers must match W."""
    import torch
    m, n, k = 2, 64, 128
    A = torch.empty((m, k), dtype=torch.bfloat16)
    Wq = torch.empty((n, k // 2), dtype=torch.uint8)
    Ws = torch.empty((n, k // 16), dtype=torch.uint8)
    g = torch.empty(1)
    out = torch.empty((m, n), dtype=torch.bfloat16)
    assert fi._mm_shapes(A, Wq, Ws, g, out) == (m, n, k)
    assert fi._mm_shapes(A, Wq, Ws, g, None) == (m, n, k)
    for bad in (torch.empty((m, n - 1), dtype=torch.bfloat16), torch.empty((m + 1, n), dtype=torch.bfloat16)):
        with pytest.raises(ValueError, match="out must be"):
            fi._mm_shapes(A, Wq, Ws, g, bad)
    with pytest.raises(ValueError, match="shape mismatch"):
        fi._mm_shapes(A, Wq, torch.empty((n, k // 32), dtype=torch.uint8), g, out)
    with pytest.raises(ValueError, match="shape mismatch"):
        fi._mm_shapes(A, torch.empty((n, k), dtype=torch.uint8), Ws, g, out)
    with pytest.raises(ValueError, match="gscale"):
        fi._mm_shapes(A, Wq, Ws, torch.empty(2), out)
    with pytest.raises(ValueError, match="is on cuda:1"):
        fi._mm_shapes(_OnDevice(A, 0), _OnDevice(Wq, 1), _OnDevice(Ws, 0), _OnDevice(g, 0), None)
    with pytest.raises(ValueError, match="out is on cuda:1"):
        fi._mm_shapes(_OnDevice(A, 0), _OnDevice(Wq, 0), _OnDevice(Ws, 0), _OnDevice(g, 0), _OnDevice(out, 1))
    W = torch.empty((n, k))
    assert fi._pack_out_check(W, (Wq, Ws, g)) == (Wq, Ws, g)
    for bad in [(Wq, Ws), (Wq[:, :-1], Ws, g), (Wq, Ws.to(torch.int8), g), (Wq, Ws, torch.empty(2)),
                (Wq, Ws, torch.empty(1, dtype=torch.float64))]:
        with pytest.raises(ValueError):
            fi._pack_out_check(W, bad)


def _tuned_entries():
    """The rows of the generated default-tactic table (csrc/tactic_table.inc)."""
    import os
    import re
    path = os.path.join(os.path.dirname(fi.__file__), "csrc", "tactic_table.inc")
    text = open(path).read()
    rows = re.findall(r"\{(\d+), (\d+), (\d+), (\d+), (\d+), (0x[0-9a-f]+), ([0-9.]+)\}", text)
    return [tuple(int(v, 0) for v in r[:6]) for r in rows if int(r[0]) > 0]


def test_tuned_table_picks_are_the_defaults_and_valid_for_their_whole_bucket():
    """Every generated entry is what the default resolves to for its (n, k, SMs) at every m of its
    bucket, it resolves at every such m, and its K split does not change inside the bucket (so
    the default stays batch-invariant within it)."""
    for n, k, m_lo, m_hi, sms, t in _tuned_entries():
        splits = set()
        for m in sorted({m_lo, (m_lo + m_hi) // 2, m_hi} | set(range(m_lo, min(m_hi, m_lo + 4) + 1))):
            assert fi.default_tactic(m, n, k, sms) == t, (n, k, m)
            splits.add(fi.resolve_tactic(m, n, k, t, sms)["splits"])
        assert len(splits) == 1, (n, k, m_lo, m_hi, splits)


def test_tuned_table_covers_every_m_once_per_shape():
    """For every (n, k, SMs) the generated table lists, its buckets are the tuner's buckets and
    tile m = 1..256 without gaps or overlaps, and the file was written by the tuner (its header)."""
    import os
    from bf16_activations_nvfp4_b200 import tune
    path = os.path.join(os.path.dirname(fi.__file__), "csrc", "tactic_table.inc")
    assert open(path).readline().startswith("// Default-tactic table: GENERATED by")
    by_shape = {}
    for n, k, m_lo, m_hi, sms, t in _tuned_entries():
        by_shape.setdefault((n, k, sms), []).append((m_lo, m_hi))
    assert by_shape
    want = [(lo, hi) for lo, hi, _ in tune.BUCKETS]
    for key, buckets in by_shape.items():
        assert sorted(buckets) == want, (key, sorted(buckets))
        assert want[0][0] == 1 and want[-1][1] == 256
        assert all(a[1] + 1 == b[0] for a, b in zip(want, want[1:]))


def test_mma_resident_activations_fit_rule():
    """Resident activations (variant 2): the largest split's slice, ceil(k/64 / S) steps of
    m_pad rows x 128 bytes, plus the raw-code ring, the row scales and the barriers must fit the
    226 KB of dynamic shared memory the kernel asks for; m_pad <= 128. The automatic variant
    takes it for one-wave grids (tiles x S <= SMs) with m <= 8 and at most 28 steps per split,
    where the B200 measurements favour it."""
    ring = 1024 + 4 * 256 * 32
    for m, n, k, S in [(8, 4096, 14336, 0), (32, 4096, 14336, 8), (1, 4096, 4096, 1), (16, 4096, 6144, 1),
                       (16, 4096, 6208, 1), (64, 152064, 5120, 1), (128, 4096, 14336, 16), (112, 2048, 7168, 4),
                       (16, 152064, 5120, 1), (8, 40000, 4096, 1), (32, 5120, 17408, 7), (8, 4096, 4096, 8),
                       (12, 4096, 4096, 4), (8, 4096, 4096, 0), (4, 14336, 4096, 8), (8, 2048, 1024, 1)]:
        info = fi.resolve_tactic(m, n, k, fi.make_tactic(fi.KIND_MMA, S, 0, 0), B200_SMS)
        m_pad = -(-m // 16) * 16
        steps = -(-(k // 64) // info["splits"])
        need = ring + steps * m_pad * 128 + -(-m_pad * 4 // 16) * 16 + 23 * 8
        fits = m_pad <= 128 and need <= 226 * 1024
        auto = fits and info["grid_x"] * info["splits"] <= B200_SMS and m <= 8 and steps <= 28
        assert info["variant"] == (2 if auto else 1), (m, n, k, S, need)
        if auto:
            assert info["smem_bytes"] == need
        explicit = fi.make_tactic(fi.KIND_MMA, info["splits"], 0, 2)
        if fits:
            assert fi.resolve_tactic(m, n, k, explicit, B200_SMS)["smem_bytes"] == need
        else:
            with pytest.raises(fi.FiError):
                fi.resolve_tactic(m, n, k, explicit, B200_SMS)

