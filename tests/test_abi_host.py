"""Host-side checks of libcpattn that need no GPU: the library loads, exports every
entry point include/cpattn.h declares, computes layout ranges and tile classes
that match the oracle's integer maps bit for bit, and rejects bad arguments
synchronously (before any CUDA call)."""
import ctypes
import os
import re

import pytest

from oracle import layout as L

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def cp():
    from context_attention_cp_b200 import build
    build.build()
    import context_attention_cp_b200 as m
    m.lib()
    return m


def _declared_symbols():
    with open(os.path.join(ROOT, "include", "cpattn.h")) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(cp_[a-z_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(cp):
    names = _declared_symbols()
    assert len(names) >= 10
    handle = ctypes.CDLL(cp.lib_path)
    for n in names:
        assert hasattr(handle, n), n
    assert cp.lib().cp_abi_version() == 1


def test_debug_library_exports_the_same_symbols(cp):
    """The bounds-checking build (libcpattn_debug.so) is the same ABI."""
    from context_attention_cp_b200 import build
    path = build.build(debug_bounds=True)
    handle = ctypes.CDLL(path)
    for n in _declared_symbols():
        assert hasattr(handle, n), n


def test_status_strings(cp):
    for code in range(7):
        assert cp.lib().cp_status_string(code)
    assert b"bounds" in cp.lib().cp_status_string(6)
    assert cp.lib().cp_status_string(99) == b"unknown status"


@pytest.mark.parametrize("layout", L.LAYOUTS)
@pytest.mark.parametrize("N,S", [(1, 16), (2, 16), (4, 64), (8, 256), (3, 24)])
def test_layout_range_matches_oracle(cp, layout, N, S):
    for rank in range(N):
        starts, lens, stride = cp.layout_range(layout, N, S, rank)
        pos = []
        for s0, n in zip(starts, lens):
            pos.extend(s0 + t * stride for t in range(n))
        assert pos == L.rank_positions(layout, N, S, rank)


def test_layout_range_random_sizes_match_oracle(cp):
    """cp_layout_range against the oracle's integer maps for random rank counts
    (1-16) and sequence lengths (multiples of N, of 2N for zig-zag); together the
    ranks' positions are a permutation of 0 .. S-1."""
    from hypothesis import given, settings
    from hypothesis import strategies as st

    @settings(max_examples=200, deadline=None)
    @given(layout=st.sampled_from(L.LAYOUTS), N=st.integers(1, 16), m=st.integers(1, 40))
    def check(layout, N, m):
        S = m * N * (2 if layout == "zigzag" else 1)
        seen = []
        for rank in range(N):
            got = _range_positions(cp.layout_range(layout, N, S, rank))
            assert got == L.rank_positions(layout, N, S, rank), (layout, N, S, rank)
            seen.extend(got)
        assert sorted(seen) == list(range(S))

    check()


def test_layout_range_rejects(cp):
    with pytest.raises(cp.CPError) as e:
        cp.layout_range("contiguous", 3, 10, 0)
    assert e.value.code == 3
    with pytest.raises(cp.CPError):
        cp.layout_range("zigzag", 4, 12, 0)
    with pytest.raises(cp.CPError):
        cp.layout_range("striped", 4, 16, 4)


def _brute_classes(pq, pk, causal, tq, tk):
    out = []
    for q0 in range(0, len(pq), tq):
        row = []
        qs = pq[q0:q0 + tq]
        for k0 in range(0, len(pk), tk):
            ks = pk[k0:k0 + tk]
            vis = sum(1 for a in qs for b in ks if (not causal) or b <= a)
            whole = len(ks) == tk
            if vis == 0:
                row.append(0)
            elif vis == len(qs) * len(ks) and whole:
                row.append(1)
            else:
                row.append(2)
        out.append(row)
    return out


@pytest.mark.parametrize("layout", L.LAYOUTS)
@pytest.mark.parametrize("N,S,tile", [(2, 64, 8), (4, 128, 8), (4, 96, 16), (3, 48, 5), (8, 256, 16)])
@pytest.mark.parametrize("causal", [True, False])
def test_tile_classes_match_brute_force(cp, layout, N, S, tile, causal):
    if layout == "zigzag" and S % (2 * N):
        pytest.skip("zig-zag needs S % 2N == 0")
    c = S // N
    for i in range(N):
        for j in range(N):
            qr, kr = cp.layout_range(layout, N, S, i), cp.layout_range(layout, N, S, j)
            got = cp.tile_classes(qr, c, kr, c, causal, tile, tile)
            want = _brute_classes(L.rank_positions(layout, N, S, i), L.rank_positions(layout, N, S, j),
                                  causal, tile, tile)
            assert got == want, (i, j)


def _random_range(draw_int, nseg):
    """An increasing position map of one or two segments (the ABI's requirement)."""
    stride = draw_int(1, 4)
    len0, start0 = draw_int(1, 70), draw_int(0, 200)
    if nseg == 1:
        return (start0,), (len0,), stride
    len1, gap = draw_int(1, 70), draw_int(1, 100)
    return (start0, start0 + (len0 - 1) * stride + gap), (len0, len1), stride


def _range_positions(r):
    starts, lens, stride = r
    return [s0 + t * stride for s0, n in zip(starts, lens) for t in range(n)]


def test_tile_classes_of_random_ranges_match_brute_force(cp):
    """The tile classifier the kernels walk with (FULL prefix, PARTIAL band, SKIP
    rest), on random increasing position maps of one or two segments, strides 1-4,
    ragged lengths and unequal query / key tile sizes, causal or not, against a
    pair-by-pair brute force."""
    from hypothesis import HealthCheck, given, settings
    from hypothesis import strategies as st

    @settings(max_examples=300, deadline=None, suppress_health_check=[HealthCheck.too_slow])
    @given(data=st.data(), nq=st.integers(1, 2), nk=st.integers(1, 2), causal=st.booleans(),
           tq=st.sampled_from([16, 32, 64, 128]), tk=st.sampled_from([16, 32, 64, 128]))
    def check(data, nq, nk, causal, tq, tk):
        draw_int = lambda lo, hi: data.draw(st.integers(lo, hi))  # noqa: E731
        qr, kr = _random_range(draw_int, nq), _random_range(draw_int, nk)
        pq, pk = _range_positions(qr), _range_positions(kr)
        got = cp.tile_classes(qr, len(pq), kr, len(pk), causal, tq, tk)
        assert got == _brute_classes(pq, pk, causal, tq, tk), (qr, kr, causal, tq, tk)

    check()


def test_tile_classes_zigzag_rectangles(cp):
    """Off-diagonal zig-zag steps need no mask: with tiles that divide c/2, no tile is
    partial unless j == i (section Zig-zag, the remark after the case table)."""
    N, S = 4, 512
    c = S // N
    for i in range(N):
        for j in range(N):
            cls = cp.tile_classes(cp.layout_range("zigzag", N, S, i), c, cp.layout_range("zigzag", N, S, j), c,
                                  True, 16, 16)
            partial = sum(x == 2 for row in cls for x in row)
            assert (partial > 0) == (i == j)


class _FakeTensor:
    """Stands in for a CUDA tensor in argument-validation tests (never dereferenced)."""


def _ct(cp, shape, dtype=0, data=0x10000, stride=None):
    from context_attention_cp_b200._binding import CpTensor
    t = CpTensor()
    t.data = data
    t.dtype = dtype
    if stride is None:
        stride = [0, 0, 0, 1]
        acc = 1
        for i in (3, 2, 1, 0):
            stride[i] = acc
            acc *= shape[i]
    for i in range(4):
        t.shape[i] = shape[i]
        t.stride[i] = stride[i]
    return t


def _call_ring(cp, q, k, v, o, lse, layout=0, N=2, causal=1, scale=0.1, mode=0):
    return cp.lib().cp_ring_attn_fwd(layout, N, causal, ctypes.byref(q), ctypes.byref(k), ctypes.byref(v),
                                     ctypes.c_float(scale), ctypes.byref(o), ctypes.byref(lse), mode, None, 0, None)


def test_ring_argument_errors_are_synchronous(cp):
    q = _ct(cp, [1, 256, 4, 128])
    k = _ct(cp, [1, 256, 2, 128])
    v = _ct(cp, [1, 256, 2, 128])
    o = _ct(cp, [1, 256, 4, 128])
    lse = _ct(cp, [1, 4, 256, 1], dtype=1)
    assert _call_ring(cp, q, k, v, o, lse, N=3) == 3            # S % N
    assert _call_ring(cp, q, k, v, o, lse, layout=1, N=3) == 3  # S % 2N
    assert _call_ring(cp, q, k, v, o, lse, layout=7) == 1       # layout
    assert _call_ring(cp, q, k, v, o, lse, scale=-1.0) == 1     # scale
    assert _call_ring(cp, q, k, v, o, lse, mode=5) == 1         # mode
    k3 = _ct(cp, [1, 256, 3, 128])
    assert _call_ring(cp, q, k3, k3, o, lse) == 3               # Hq % Hkv
    q96 = _ct(cp, [1, 256, 4, 96])
    assert _call_ring(cp, q96, k, v, o, lse) in (2, 3)          # head dim
    kf = _ct(cp, [1, 256, 2, 128], dtype=1)
    assert _call_ring(cp, q, kf, kf, o, lse) == 1               # mixed dtypes
    bad = _ct(cp, [1, 256, 4, 128], data=0x10008)
    assert _call_ring(cp, bad, k, v, o, lse) == 1               # alignment
    lse_bad = _ct(cp, [1, 4, 255, 1], dtype=1)
    assert _call_ring(cp, q, k, v, o, lse_bad) == 3             # lse shape
    assert b"multiple" in cp.lib().cp_last_error() or cp.lib().cp_last_error()


def test_block_argument_errors_are_synchronous(cp):
    from context_attention_cp_b200._binding import CpRange
    q = _ct(cp, [1, 128, 2, 64], dtype=1)
    k = _ct(cp, [1, 100, 2, 64], dtype=1)
    o = _ct(cp, [1, 128, 2, 64], dtype=1)
    lse = _ct(cp, [1, 2, 128, 1], dtype=1)
    qr, kr = CpRange(), CpRange()
    qr.nseg, qr.start[0], qr.len[0], qr.stride = 1, 0, 128, 1
    kr.nseg, kr.start[0], kr.len[0], kr.stride = 1, 0, 99, 1  # wrong length
    f = cp.lib().cp_block_attn_fwd
    assert f(ctypes.byref(q), ctypes.byref(k), ctypes.byref(k), ctypes.byref(qr), ctypes.byref(kr), 1,
             ctypes.c_float(0.1), ctypes.byref(o), ctypes.byref(lse), 0, None) == 3
    kr.len[0] = 100
    kr.nseg, kr.start[1], kr.len[0], kr.len[1] = 2, 10, 50, 50  # second segment overlaps the first
    assert f(ctypes.byref(q), ctypes.byref(k), ctypes.byref(k), ctypes.byref(qr), ctypes.byref(kr), 1,
             ctypes.c_float(0.1), ctypes.byref(o), ctypes.byref(lse), 0, None) == 1
    kr.nseg, kr.len[0] = 1, 100
    o16 = _ct(cp, [1, 128, 2, 64], dtype=0)
    assert f(ctypes.byref(q), ctypes.byref(k), ctypes.byref(k), ctypes.byref(qr), ctypes.byref(kr), 1,
             ctypes.c_float(0.1), ctypes.byref(o16), ctypes.byref(lse), 0, None) == 1  # fp32 in -> fp32 out
    assert f(ctypes.byref(q), ctypes.byref(k), ctypes.byref(k), ctypes.byref(qr), ctypes.byref(kr), 1,
             ctypes.c_float(0.1), ctypes.byref(o16), ctypes.byref(lse), 1, None) == 1  # accumulate needs fp32


def test_merge_and_permute_argument_errors(cp):
    oa = _ct(cp, [1, 16, 2, 128], dtype=1)
    ob = _ct(cp, [1, 16, 2, 128], dtype=0)
    la = _ct(cp, [1, 2, 16, 1], dtype=1)
    lb = _ct(cp, [1, 2, 16, 1], dtype=1)
    f = cp.lib().cp_lse_merge
    ob_bad = _ct(cp, [1, 16, 3, 128], dtype=0)
    assert f(ctypes.byref(oa), ctypes.byref(la), ctypes.byref(ob_bad), ctypes.byref(lb), None, None) == 3
    oa16 = _ct(cp, [1, 16, 2, 128], dtype=0)
    assert f(ctypes.byref(oa16), ctypes.byref(la), ctypes.byref(ob), ctypes.byref(lb), None, None) == 1
    x = _ct(cp, [1, 16, 2, 128], dtype=0)
    y = _ct(cp, [1, 16, 2, 128], dtype=0, data=0x20000)
    g = cp.lib().cp_layout_permute
    assert g(1, 3, 1, ctypes.byref(x), ctypes.byref(y), 0, None) == 3       # 16 % 6
    assert g(0, 2, 1, ctypes.byref(x), ctypes.byref(x), 0, None) == 1       # overlap
    assert cp.lib().cp_ring_workspace_bytes(0, 4, 0, 0, 1, 256, 4, 128) == 0  # fused needs none
    assert cp.lib().cp_ring_workspace_bytes(0, 4, 1, 0, 1, 256, 4, 128) >= 256 * 4 * 128 * 6


def test_selftest_limit_is_checked_before_any_launch(cp):
    f = cp.lib().cp_selftest_wait_timeout
    assert f(10, None) == 1             # below 1 ms
    assert f(5_000_000_000, None) == 1  # above 1 s


def test_ring_bwd_argument_errors_are_synchronous(cp):
    q = _ct(cp, [1, 256, 4, 128])
    k = _ct(cp, [1, 256, 2, 128])
    o = _ct(cp, [1, 256, 4, 128])
    lse = _ct(cp, [1, 4, 256, 1], dtype=1)
    dq = _ct(cp, [1, 256, 4, 128])
    dk = _ct(cp, [1, 256, 2, 128])
    f = cp.lib().cp_ring_attn_bwd
    need = cp.lib().cp_ring_bwd_workspace_bytes(1, 2, 0, 1, 256, 4, 128)
    assert need >= 256 * 4 * 128 * 4      # the fp32 dQ accumulator at least

    def call(layout=1, N=2, causal=1, q_=q, k_=k, o_=o, lse_=lse, do_=q, dq_=dq, dk_=dk, ws=0x100000, wsb=None):
        return f(layout, N, causal, ctypes.byref(q_), ctypes.byref(k_), ctypes.byref(k_), ctypes.byref(o_),
                 ctypes.byref(lse_), ctypes.byref(do_), ctypes.c_float(0.088), ctypes.byref(dq_), ctypes.byref(dk_),
                 ctypes.byref(dk_), ctypes.c_void_p(ws), need if wsb is None else wsb, None)

    assert call(N=3) == 3                                  # S % 2N
    assert call(layout=9) == 1                             # layout
    assert call(causal=2) == 1                             # causal flag
    assert call(wsb=16) == 1                               # workspace too small
    assert call(ws=0x100010) == 1                          # workspace alignment
    assert call(q_=_ct(cp, [1, 256, 4, 256]), k_=_ct(cp, [1, 256, 2, 256])) == 2  # d = 256 unsupported
    qf = _ct(cp, [1, 256, 4, 128], dtype=1)
    assert call(q_=qf, k_=_ct(cp, [1, 256, 2, 128], dtype=1)) == 1             # fp32 q with a bf16 o
    assert call(q_=qf, k_=_ct(cp, [1, 256, 2, 128], dtype=1), o_=_ct(cp, [1, 256, 4, 128], dtype=1),
                do_=qf) == 3                                                    # bf16 dq for fp32 q
    assert call(dk_=_ct(cp, [1, 256, 4, 128])) == 3        # dk shaped like q
    assert call(lse_=_ct(cp, [1, 4, 255, 1], dtype=1)) == 3
    assert cp.lib().cp_ring_bwd_workspace_bytes(1, 3, 0, 1, 256, 4, 128) == 0  # S % N


def test_allgather_argument_errors_are_synchronous(cp):
    q = _ct(cp, [1, 256, 4, 128])
    k = _ct(cp, [1, 256, 2, 128])
    o = _ct(cp, [1, 256, 4, 128])
    lse = _ct(cp, [1, 4, 256, 1], dtype=1)
    f = cp.lib().cp_allgather_attn_fwd
    need = cp.lib().cp_allgather_workspace_bytes(2, 0, 1, 256, 2, 128, 3)
    assert need >= 2 * 256 * 2 * 128 * 2

    def call(docs, layout=1, N=2, causal=1, q_=q, k_=k, ws=0x100000, wsb=None):
        arr = (ctypes.c_int64 * len(docs))(*docs)
        return f(layout, N, causal, ctypes.byref(q_), ctypes.byref(k_), ctypes.byref(k_), arr, len(docs),
                 ctypes.c_float(0.088), ctypes.byref(o), ctypes.byref(lse), ctypes.c_void_p(ws),
                 need if wsb is None else wsb, None)

    assert call([1, 10]) == 1                    # first document must start at 0
    assert call([0, 10, 10]) == 1                # strictly increasing
    assert call([0, 256]) == 1                   # below S
    assert call([0, 100], causal=0) == 2         # document mask needs the causal mask
    assert call([0, 100], N=3) == 3              # S % 2N
    assert call([0, 100], wsb=64) == 1           # workspace too small
    assert call([0, 100], ws=0x100040) == 1      # workspace alignment
    qf, kf = _ct(cp, [1, 256, 4, 128], dtype=1), _ct(cp, [1, 256, 2, 128], dtype=1)
    assert call([0], q_=qf, k_=kf) == 1          # fp32 q with a bf16 o
    q256, k256 = _ct(cp, [1, 256, 4, 256]), _ct(cp, [1, 256, 2, 256])
    assert call([0], q_=q256, k_=k256) == 2      # head dim 256
    assert cp.lib().cp_allgather_workspace_bytes(2, 0, 1, 256, 2, 128, 0) == 0


def test_ulysses_argument_errors_are_synchronous(cp):
    x = _ct(cp, [1, 64, 8, 128])
    y = _ct(cp, [4, 64, 2, 128], data=0x200000)
    g = cp.lib().cp_ulysses_all_to_all
    assert g(4, 2, ctypes.byref(x), ctypes.byref(y), None) == 1      # direction
    assert g(3, 0, ctypes.byref(x), ctypes.byref(y), None) == 3      # P divides H
    y_bad = _ct(cp, [4, 64, 4, 128], data=0x200000)
    assert g(4, 0, ctypes.byref(x), ctypes.byref(y_bad), None) == 3  # y shape
    y_ov = _ct(cp, [4, 64, 2, 128], data=0x10000)
    assert g(4, 0, ctypes.byref(x), ctypes.byref(y_ov), None) == 1   # overlap
    q = _ct(cp, [1, 64, 8, 128])
    k = _ct(cp, [1, 64, 2, 128])
    o = _ct(cp, [1, 64, 8, 128])
    lse = _ct(cp, [1, 8, 64, 1], dtype=1)
    f = cp.lib().cp_ulysses_attn_fwd
    assert f(4, 1, ctypes.byref(q), ctypes.byref(k), ctypes.byref(k), ctypes.c_float(0.1), ctypes.byref(o),
             ctypes.byref(lse), ctypes.c_void_p(0x100000), 1 << 30, None) == 3   # P must divide Hkv = 2
    assert f(2, 1, ctypes.byref(q), ctypes.byref(k), ctypes.byref(k), ctypes.c_float(0.1), ctypes.byref(o),
             ctypes.byref(lse), ctypes.c_void_p(0x100000), 16, None) == 1        # workspace too small
    assert cp.lib().cp_ulysses_workspace_bytes(0, 0, 1, 64, 8, 2, 128) == 0


def test_usp_argument_errors_are_synchronous(cp):
    q = _ct(cp, [1, 64, 8, 128])
    k = _ct(cp, [1, 64, 2, 128])
    o = _ct(cp, [1, 64, 8, 128])
    lse = _ct(cp, [1, 8, 64, 1], dtype=1)
    f = cp.lib().cp_usp_attn_fwd

    def call(layout, N, P, q_=q, k_=k, o_=o, lse_=lse, wsb=1 << 30):
        return f(layout, N, P, 1, ctypes.byref(q_), ctypes.byref(k_), ctypes.byref(k_), ctypes.c_float(0.1),
                 ctypes.byref(o_), ctypes.byref(lse_), ctypes.c_void_p(0x100000), wsb, None)

    assert call(7, 2, 2) == 1                 # layout
    assert call(1, 0, 2) == 1                 # N >= 1
    assert call(1, 2, 4) == 3                 # P must divide Hkv = 2
    assert call(0, 3, 2) == 3                 # S % (N P)
    assert call(1, 2, 2, wsb=16) == 1         # workspace too small
    q12, k12 = _ct(cp, [1, 12, 8, 128]), _ct(cp, [1, 12, 2, 128])
    o12, l12 = _ct(cp, [1, 12, 8, 128]), _ct(cp, [1, 8, 12, 1], dtype=1)
    assert call(1, 4, 1, q12, k12, o12, l12) == 3    # zig-zag: S % 2N
    assert cp.lib().cp_usp_workspace_bytes(5, 2, 2, 0, 1, 64, 8, 2, 128) == 0
    assert cp.lib().cp_usp_bwd_workspace_bytes(0, 3, 2, 0, 1, 64, 8, 2, 128) == 0   # S % N
    assert cp.lib().cp_usp_bwd_workspace_bytes(0, 2, 2, 0, 1, 64, 8, 2, 128) > 0
    g = cp.lib().cp_usp_attn_bwd
    qf, kf = _ct(cp, [1, 64, 8, 128], dtype=1), _ct(cp, [1, 64, 2, 128], dtype=1)
    of = _ct(cp, [1, 64, 8, 128], dtype=1)
    assert g(1, 2, 2, 1, *[ctypes.byref(t) for t in (qf, kf, kf, of, lse, of)], ctypes.c_float(0.1),
             *[ctypes.byref(t) for t in (q, kf, kf)], ctypes.c_void_p(0x100000), 1 << 30, None) == 3  # dq dtype


@pytest.mark.parametrize("b,S", [(0, 256), (1, 0)])
def test_empty_inputs_return_ok_without_device_work(cp, b, S):
    """Empty batches or sequences are valid and launch nothing: on this host (no
    device) any launch or device query would come back as CP_ERR_CUDA."""
    L = cp.lib()
    q = _ct(cp, [b, S, 4, 128])
    k = _ct(cp, [b, S, 2, 128], data=0x20000)
    o = _ct(cp, [b, S, 4, 128], data=0x30000)
    lse = _ct(cp, [b, 4, S, 1], dtype=1, data=0x40000)
    ws = ctypes.c_void_p(0x100000)
    r = lambda *ts: [ctypes.byref(t) for t in ts]  # noqa: E731
    sc = ctypes.c_float(0.1)
    docs = (ctypes.c_int64 * 1)(0)
    calls = {
        "ring_fwd": L.cp_ring_attn_fwd(1, 2, 1, *r(q, k, k), sc, *r(o, lse), 0, ws, 1 << 30, None),
        "ring_bwd": L.cp_ring_attn_bwd(1, 2, 1, *r(q, k, k, o, lse, q), sc, *r(o, k, k), ws, 1 << 30, None),
        "allgather_fwd": L.cp_allgather_attn_fwd(1, 2, 1, *r(q, k, k), docs, 1, sc, *r(o, lse), ws, 1 << 30, None),
        "allgather_bwd": L.cp_allgather_attn_bwd(1, 2, 1, *r(q, k, k, o, lse, q), docs, 1, sc, *r(o, k, k), ws,
                                                 1 << 30, None),
        "ulysses_fwd": L.cp_ulysses_attn_fwd(2, 1, *r(q, k, k), sc, *r(o, lse), ws, 1 << 30, None),
        "ulysses_bwd": L.cp_ulysses_attn_bwd(2, 1, *r(q, k, k, o, lse, q), sc, *r(o, k, k), ws, 1 << 30, None),
        "usp_fwd": L.cp_usp_attn_fwd(1, 2, 2, 1, *r(q, k, k), sc, *r(o, lse), ws, 1 << 30, None),
        "usp_bwd": L.cp_usp_attn_bwd(1, 2, 2, 1, *r(q, k, k, o, lse, q), sc, *r(o, k, k), ws, 1 << 30, None),
        "permute": L.cp_layout_permute(1, 2, 1, *r(q, o), 0, None),
    }
    assert all(v == 0 for v in calls.values()), calls


def test_block_bwd_argument_errors_are_synchronous(cp):
    from context_attention_cp_b200._binding import _range
    L = cp.lib()
    q, o, do = _ct(cp, [1, 128, 4, 64]), _ct(cp, [1, 128, 4, 64], data=0x30000), _ct(cp, [1, 128, 4, 64], data=0x50000)
    k = _ct(cp, [1, 96, 2, 64], data=0x20000)
    lse = _ct(cp, [1, 4, 128, 1], dtype=1, data=0x40000)
    dq = _ct(cp, [1, 128, 4, 64], dtype=1, data=0x60000)
    dk = _ct(cp, [1, 96, 2, 64], dtype=1, data=0x70000)
    qr, kr = _range(((0,), (128,), 1)), _range(((0,), (96,), 1))
    need = L.cp_block_bwd_workspace_bytes(1, 128, 4)
    assert need >= 128 * 4 * 8

    def call(mask=1, dq_=dq, dk_=dk, wsb=None, ws=0x100000, kr_=kr):
        return L.cp_block_attn_bwd(ctypes.byref(q), ctypes.byref(k), ctypes.byref(k), ctypes.byref(o), ctypes.byref(lse),
                                   ctypes.byref(do), ctypes.byref(qr), ctypes.byref(kr_), mask, ctypes.c_float(0.125),
                                   ctypes.byref(dq_), ctypes.byref(dk_), ctypes.byref(dk_), ctypes.c_void_p(ws),
                                   need if wsb is None else wsb, None)

    assert call(mask=3) == 1                                   # mask mode
    assert call(dq_=_ct(cp, [1, 128, 4, 64], data=0x60000)) == 3   # bf16 accumulator
    assert call(dk_=_ct(cp, [1, 96, 4, 64], dtype=1, data=0x70000)) == 3   # dk shaped like q
    assert call(wsb=8) == 1                                    # workspace too small
    assert call(ws=0x100008) == 1                              # workspace alignment
    assert call(kr_=_range(((0,), (95,), 1))) != 0             # range length differs from the key block


def test_peer_calls_reject_null_arguments(cp):
    """cp_peer_export / cp_peer_import / cp_peer_close / cp_peer_copy refuse NULL
    arguments before any CUDA call; the handle struct has the layout the header
    declares."""
    from context_attention_cp_b200._binding import CpPeerHandle
    assert ctypes.sizeof(CpPeerHandle) == 64 + 8 + 8
    h = CpPeerHandle()
    assert cp.lib().cp_peer_export(None, ctypes.byref(h)) == 1
    assert cp.lib().cp_peer_export(ctypes.c_void_p(0x1000), None) == 1
    assert cp.lib().cp_peer_import(None, ctypes.byref(ctypes.c_void_p())) == 1
    assert cp.lib().cp_peer_import(ctypes.byref(h), None) == 1
    assert cp.lib().cp_peer_close(None) == 1
    assert b"NULL" in cp.lib().cp_last_error()
    assert cp.lib().cp_peer_copy(None, ctypes.c_void_p(0x1000), 16, None) == 1
    assert cp.lib().cp_peer_copy(None, None, 0, None) == 0   # nothing to copy: no CUDA call


def test_peer_import_checks_size_and_dtype_before_mapping(cp):
    """peer_import refuses a view larger than the exported block and an unsupported
    dtype before it maps anything (no CUDA call)."""
    import torch

    from context_attention_cp_b200._binding import CpPeerHandle
    h = CpPeerHandle()
    h.offset, h.bytes = 0, 64
    with pytest.raises(ValueError):
        cp.peer_import(bytes(h), (1, 16, 1, 2), torch.float32)      # 128 bytes asked, 64 held
    with pytest.raises(TypeError):
        cp.peer_import(bytes(h), (1, 4, 1, 2), torch.float16)


def test_allgather_workspace_holds_the_pages_full_kv_bytes(cp):
    """The gathered K/V term of cp_allgather_workspace_bytes equals the page's full
    K/V size (512 MiB for the 70B heads at 128K, 64 MiB with one KV head).  The rest
    of the workspace (document tables) does not depend on n_kv, so the K/V term of
    n_kv heads is (ws(n_kv) - ws(1)) * n_kv / (n_kv - 1) and that of one head
    ws(n_kv) - ws(1) over n_kv - 1."""
    rows = []
    with open(os.path.join(ROOT, "tests", "golden", "allgather_kv_bytes.txt")) as f:
        for ln in f:
            if ln.strip() and not ln.startswith("#"):
                rows.append([int(x) for x in ln.split()])
    assert len(rows) == 2
    (b, S, hkv, d, want8), (_, _, one, _, want1) = rows
    assert one == 1
    ws = {h: cp.allgather_workspace_bytes(8, 0, b, S, h, d, 1) for h in (1, hkv)}
    per_head = (ws[hkv] - ws[1]) // (hkv - 1)
    assert (ws[hkv] - ws[1]) % (hkv - 1) == 0
    assert per_head * hkv == want8 == 2 * 2 * b * S * hkv * d
    assert per_head == want1

