"""GPU parity: every libsq stage against the CPU oracle on the same seeded inputs (through the C ABI).

Bars (the tolerances stated for the method, written here in the tests):
  * abs-maxima, INT8 codes, per-row scales and INT32 accumulators: bit-exact;
  * smoothing factors and fold: within 1e-6 relative (the device pow is not correctly rounded);
  * bf16 outputs: within 1e-2 relative of the exact dequantised value, and in practice bit-exact
    against the oracle's epilogue, which takes the same binary32 steps.
Each later stage is fed the GPU's own earlier outputs on both sides, so a tolerance at one stage
cannot cascade into code mismatches downstream.
All five workloads run at their full sizes in the launch configuration the benchmark uses; the GEMM
is checked on sampled full output rows and full output columns (the oracle computes those one by
one), the other stages on every element.
"""
import os

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

from post_quantization_calib_b200 import synth  # noqa: E402

# SQ_CHECKED=1: run against libsq_checked.so, the kernels with device-side bounds checks compiled in
CHECKED = os.environ.get("SQ_CHECKED", "0") not in ("", "0")
SQ_ERR_BOUNDS = 7


@pytest.fixture(scope="module")
def sq():
    from post_quantization_calib_b200 import build
    build.build(checked=CHECKED)
    from post_quantization_calib_b200 import sq as m
    assert m.CHECKED == CHECKED
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return m


@pytest.fixture(autouse=True)
def no_failed_bounds_check():
    """Under the checked library, no test may leave a failed device-side bounds check behind."""
    yield
    if CHECKED:
        from post_quantization_calib_b200 import sq as m
        st = m.sq_device_status()
        assert st != SQ_ERR_BOUNDS, "a device-side bounds check failed (SQ_ERR_BOUNDS)"


def h16(t):
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def hnp(t):
    return None if t is None else t.detach().contiguous().cpu().numpy()


def f64(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def ok_status(sq):
    st = sq.sq_device_status()
    assert st == 0, f"device status {sq.sq_status_string(st)}"


def check_linear(sq, orc, xq, xs, wq, ws, bias, y, acc, rows=None, cols=None):
    """Compare GPU accumulators and bf16 outputs with the oracle on the given rows / columns."""
    xq_h, wq_h, xs_h, ws_h = hnp(xq), hnp(wq), hnp(xs), hnp(ws)
    b_h = h16(bias) if bias is not None else None
    ri = None if rows is None else torch.as_tensor(rows, device=y.device)
    ci = None if cols is None else torch.as_tensor(cols, device=y.device)
    acc_g, y_g = acc, y
    if ri is not None:
        acc_g, y_g = acc_g.index_select(0, ri), y_g.index_select(0, ri)
    if ci is not None:
        acc_g, y_g = acc_g.index_select(1, ci), y_g.index_select(1, ci)
    acc_g, y_g = hnp(acc_g), h16(y_g)
    y_o, acc_o = orc.w8a8_linear(xq_h, xs_h, wq_h, ws_h, b_h, rows, cols)
    bad = np.argwhere(acc_g != acc_o)
    assert bad.size == 0, f"{len(bad)} accumulator mismatches, first at {bad[:3].tolist()}"
    # the stated bar: 1e-2 relative of the exact dequantised value (plus bf16-level slack near 0)
    rsel = slice(None) if rows is None else rows
    csel = slice(None) if cols is None else cols
    exact = acc_o.astype(np.float64) * xs_h[rsel][:, None].astype(np.float64) * ws_h[csel][None, :]
    bb = f64(b_h[csel])[None, :] if b_h is not None else 0.0
    ref = exact + bb
    err = np.abs(f64(y_g) - ref)
    assert np.all(err <= 1e-2 * np.abs(ref) + 1e-2 * 2.0 ** -8 * (np.abs(exact) + np.abs(bb)) + 1e-30)
    # and the same binary32 steps give the same bits
    assert np.array_equal(y_g, y_o), f"{int((y_g != y_o).sum())} bf16 outputs differ from the oracle epilogue"


def sample_indices(n, k, seed):
    rng = np.random.default_rng(seed)
    pick = set(rng.choice(n, size=min(k, n), replace=False).tolist())
    pick |= {0, n - 1, min(n - 1, 127), min(n - 1, 128), max(0, n - 129)}
    return np.array(sorted(pick), np.int64)


def run_group(sq, orc, w, g, T=None, gemm_sample=None, alphas=None):
    """Full stage-by-stage parity for smoothing group g of workload w on the GPU."""
    dev = "cuda"
    d = synth.group_inputs(w, g, dev, T=T)
    gamma, W, bias, X = d["gamma"], d["weight"], d["bias"], d["x"]
    K, N = W.shape[1], W.shape[0]
    T = X.shape[0]
    gamma_h = hnp(gamma)

    # S1: calibration abs-max, streamed in chunks with the running maximum
    amax = torch.empty(K, dtype=torch.float32, device=dev)
    amax_o = np.zeros(K, np.float32)
    for i, chunk in enumerate(synth.calibration_chunks(w, d["channels"], dev, group=g)):
        sq.sq_calibrate_absmax(chunk, norm_gamma=gamma, eps=w.eps, amax=amax, accumulate=i > 0)
        orc.calibrate_absmax(h16(chunk), norm_gamma=gamma_h, eps=w.eps, amax=amax_o, accumulate=i > 0)
    ok_status(sq)
    assert np.array_equal(hnp(amax), amax_o), "activation abs-max differs"

    # S2: weight abs-max per input channel
    aw = sq.sq_calibrate_absmax(W)
    assert np.array_equal(hnp(aw), orc.calibrate_absmax(h16(W))), "weight abs-max differs"

    # S3: smoothing factors (and the alpha sweep where the workload asks for one)
    for a in (alphas or [w.alpha]):
        s_a, f_a = sq.sq_compute_scales(amax, aw, a, gamma=gamma)
        s_o, f_o = orc.compute_scales(hnp(amax), hnp(aw), a, gamma_h)
        assert np.all(np.abs(hnp(s_a).astype(np.float64) / s_o - 1) <= 1e-6), f"s differs at alpha={a}"
        assert np.all(np.abs(hnp(f_a).astype(np.float64) / f_o - 1) <= 1e-6), f"fold differs at alpha={a}"
    s, fold = sq.sq_compute_scales(amax, aw, w.alpha, gamma=gamma)

    # S4: smoothed weight, INT8 per output channel (oracle fed the GPU's s)
    wq, ws = sq.sq_smooth_quantize_weight(W, s)
    wq_o, ws_o = orc.smooth_quantize_weight(h16(W), hnp(s))
    assert np.array_equal(hnp(ws), ws_o), "weight scales differ"
    assert np.array_equal(hnp(wq), wq_o), "weight codes differ"

    # S5: fused RMSNorm(gamma/s) + per-token INT8 (oracle fed the GPU's fold)
    xq, xs = sq.sq_rmsnorm_smooth_quant(X, fold, eps=w.eps, apply_norm=w.norm)
    xq_o, xs_o = orc.rmsnorm_smooth_quant(h16(X), hnp(fold), eps=w.eps, apply_norm=w.norm)
    assert np.array_equal(hnp(xs), xs_o), "token scales differ"
    assert np.array_equal(hnp(xq), xq_o), "token codes differ"

    # S6 + S7: INT8 GEMM with the dequant epilogue
    acc = torch.empty(T, N, dtype=torch.int32, device=dev)
    y = sq.sq_w8a8_linear(xq, xs, wq, ws, bias=bias, acc_out=acc)
    ok_status(sq)
    if gemm_sample is None:
        check_linear(sq, orc, xq, xs, wq, ws, bias, y, acc)
    else:
        rows = sample_indices(T, gemm_sample, 7 + g)
        cols = sample_indices(N, gemm_sample, 11 + g)
        check_linear(sq, orc, xq, xs, wq, ws, bias, y, acc, rows=rows, cols=None)
        check_linear(sq, orc, xq, xs, wq, ws, bias, y, acc, rows=None, cols=cols)
    return y


def test_single_linear_full(sq, orc):
    run_group(sq, orc, synth.WORKLOADS[0], 0)


def test_qproj_alpha_sweep(sq, orc):
    alphas = [round(0.1 * i, 1) for i in range(1, 11)]
    run_group(sq, orc, synth.WORKLOADS[1], 0, gemm_sample=40, alphas=alphas)


@pytest.mark.parametrize("g", [0, 1])
def test_block_prefill_groups(sq, orc, g):
    run_group(sq, orc, synth.WORKLOADS[2], g, gemm_sample=32)


@pytest.mark.parametrize("T", [1, 8, 32, 64])
def test_decode_shapes(sq, orc, T):
    run_group(sq, orc, synth.WORKLOADS[3], 0, T=T)


def test_mlp_up_70b(sq, orc):
    run_group(sq, orc, synth.WORKLOADS[4], 0, gemm_sample=24)


# ---------------------------------------------------------------------------------------------
# Edge cases: ragged tiles, tiny sizes, K not a multiple of the 128-byte stage, zero rows.

EDGE = [
    # T, N, K, norm, bias
    (1, 8, 16, False, False),
    (1, 264, 144, True, True),
    (129, 264, 1040, True, False),
    (300, 520, 272, False, True),
    (128, 256, 128, True, False),
    (255, 512, 4096, False, False),
    (777, 1288, 2064, True, True),
    # enough 256-channel tiles to take the wide form, with ragged T, N and K
    (2000, 2312, 1040, True, True),
    (1100, 5000, 1040, False, True),
    (2000, 4104, 1040, True, True),
    (64, 37888, 64, False, True),
    # decode form with ragged N (a partial last weight tile) and T just below its 16 / 128 buckets
    (33, 14344, 1040, True, True),
    (128, 1000, 272, False, False),
]


@pytest.mark.parametrize("T,N,K,norm,bias", EDGE)
def test_edge_shapes(sq, orc, T, N, K, norm, bias):
    dev = "cuda"
    seed = T * 7 + N * 3 + K
    ch = synth.outlier_channels(K, synth.OutlierSpec(max(1, K // 64), 10.0, 100.0), seed)
    X = synth.outlier_tokens(T, K, ch, seed + 1, dev)
    X[T // 2].zero_()                              # an all-zero token: scale 0, codes 0
    W = synth.normal_weight(N, K, seed + 2, dev)
    W[N - 1].zero_()                               # an all-zero output channel
    gamma = synth.norm_gamma(K, seed + 3, dev) if norm else None
    b = synth.bias_vector(N, seed + 4, dev) if bias else None
    amax = sq.sq_calibrate_absmax(X, norm_gamma=gamma)
    assert np.array_equal(hnp(amax), orc.calibrate_absmax(h16(X), norm_gamma=hnp(gamma)))
    aw = sq.sq_calibrate_absmax(W)
    assert np.array_equal(hnp(aw), orc.calibrate_absmax(h16(W)))
    s, fold = sq.sq_compute_scales(amax, aw, 0.5, gamma=gamma)
    wq, ws = sq.sq_smooth_quantize_weight(W, s)
    wq_o, ws_o = orc.smooth_quantize_weight(h16(W), hnp(s))
    assert np.array_equal(hnp(wq), wq_o) and np.array_equal(hnp(ws), ws_o)
    assert hnp(ws)[N - 1] == 0 and np.all(hnp(wq)[N - 1] == 0)
    xq, xs = sq.sq_rmsnorm_smooth_quant(X, fold, apply_norm=norm)
    xq_o, xs_o = orc.rmsnorm_smooth_quant(h16(X), hnp(fold), apply_norm=norm)
    assert np.array_equal(hnp(xq), xq_o) and np.array_equal(hnp(xs), xs_o)
    assert hnp(xs)[T // 2] == 0 and np.all(hnp(xq)[T // 2] == 0)
    acc = torch.empty(T, N, dtype=torch.int32, device=dev)
    y = sq.sq_w8a8_linear(xq, xs, wq, ws, bias=b, acc_out=acc)
    check_linear(sq, orc, xq, xs, wq, ws, b, y, acc)
    ok_status(sq)


# all +-127 codes: |acc| = K * 16129; K = 8192 is the widest configuration, K = 131072 the widest the GEMM
# accepts (131072 * 16129 = 2114060288 < 2^31), in the token-tile form and in the decode form (T <= 128)
@pytest.mark.parametrize("T,N,K", [(130, 264, 8192), (130, 264, 131072), (16, 264, 131072)])
def test_extreme_codes_accumulate_exactly(sq, orc, T, N, K):
    dev = "cuda"
    xq = torch.full((T, K), 127, dtype=torch.int8, device=dev)
    xq[1::2] = -127
    wq = torch.full((N, K), -127, dtype=torch.int8, device=dev)
    wq[::3] = 127
    xs = torch.full((T,), 1e-3, device=dev)
    ws = torch.full((N,), 2e-4, device=dev)
    acc = torch.empty(T, N, dtype=torch.int32, device=dev)
    y = sq.sq_w8a8_linear(xq, xs, wq, ws, acc_out=acc)
    check_linear(sq, orc, xq, xs, wq, ws, None, y, acc)
    assert int(hnp(acc).max()) == K * 16129


def test_absmax_strided_rows_and_empty(sq, orc):
    dev = "cuda"
    big = synth.outlier_tokens(100, 96, synth.outlier_channels(96, synth.OutlierSpec(3, 10, 20), 1), 2, dev)
    view = big[:, :64]                              # ld = 96, cols = 64
    a = sq.sq_calibrate_absmax(view)
    assert np.array_equal(hnp(a), np.abs(f64(h16(big))[:, :64]).max(axis=0).astype(np.float32))
    empty = big[:0, :64]
    z = torch.full((64,), 3.0, device=dev)
    sq.sq_calibrate_absmax(empty, amax=z, accumulate=True)       # running max over no rows: unchanged
    assert np.all(hnp(z) == 3.0)
    sq.sq_calibrate_absmax(empty, amax=z, accumulate=False)      # overwrite with no rows: zeros
    assert np.all(hnp(z) == 0.0)
    ok_status(sq)


# Both maxima of a smoothing group in one call, against the oracle's two reductions: the one-launch
# form (rows of more than 2048 elements, both inputs non-empty; norm-fed or plain activations; whole
# and ragged rows; strided inputs) and the two-launch form (narrow rows, one input empty), each with
# overwrite and running-maximum semantics.
PAIR_ABSMAX = [  # rows, w_rows, cols, norm, extra columns of a's row stride, of w's row stride
    (65536, 4096, 4096, True, 0, 0),      # the query projection's calibration set and weight
    (3000, 5000, 4096, True, 0, 0),       # more weight rows than activation rows
    (777, 130, 2568, True, 8, 16),        # a row that is not a whole number of lane vectors; strided
    (500, 7000, 8192, False, 0, 8),       # plain activations, wider rows
    (64, 64, 16384, True, 0, 0),          # the widest rows
    (1000, 300, 1024, True, 0, 0),        # narrow rows: two launches
    (0, 300, 4096, True, 0, 0),           # no activation rows
    (300, 0, 4096, False, 0, 0),          # no weight rows
]


@pytest.mark.parametrize("rows,w_rows,cols,norm,xa,xw", PAIR_ABSMAX)
def test_absmax_pair(sq, orc, rows, w_rows, cols, norm, xa, xw):
    dev = "cuda"
    ch = synth.outlier_channels(cols + xa, synth.OutlierSpec(max(1, cols // 64), 10, 40), 5)
    a = synth.outlier_tokens(rows, cols + xa, ch, 6, dev)[:, :cols]
    w = synth.normal_weight(w_rows, cols + xw, 7, dev)[:, :cols]
    g = synth.norm_gamma(cols, 8, dev) if norm else None
    g_h = None if g is None else hnp(g)
    ax, aw = sq.sq_calibrate_absmax_pair(a, w, norm_gamma=g, eps=1e-6)
    ok_status(sq)
    a_h, w_h = h16(a), h16(w)
    ref_a = orc.calibrate_absmax(a_h, norm_gamma=g_h, eps=1e-6)
    ref_w = orc.calibrate_absmax(w_h)
    assert np.array_equal(hnp(ax), ref_a)
    assert np.array_equal(hnp(aw), ref_w)
    # running maxima: a second batch (half the rows, scaled up) raises some columns of each output
    a2, w2 = (a[: rows // 2] * 3).contiguous(), (w[: w_rows // 2] * 3).contiguous()
    sq.sq_calibrate_absmax_pair(a2, w2, norm_gamma=g, eps=1e-6, amax=ax, amax_w=aw, accumulate=True)
    ok_status(sq)
    orc.calibrate_absmax(h16(a2), norm_gamma=g_h, eps=1e-6, amax=ref_a, accumulate=True)
    orc.calibrate_absmax(h16(w2), amax=ref_w, accumulate=True)
    assert np.array_equal(hnp(ax), ref_a)
    assert np.array_equal(hnp(aw), ref_w)


def test_absmax_pair_matches_two_calls_at_every_split(sq):
    """The one-launch form against two sq_calibrate_absmax calls over a range of input sizes, so that
    the CTA split between the inputs takes many values (including the smallest share)."""
    dev = "cuda"
    K = 4096
    ch = synth.outlier_channels(K, synth.OutlierSpec(64, 10, 40), 9)
    a_all = synth.outlier_tokens(40000, K, ch, 10, dev)
    w_all = synth.normal_weight(40000, K, 11, dev)
    g = synth.norm_gamma(K, 12, dev)
    for rows, w_rows in [(40000, 1), (40000, 40), (20000, 2000), (9000, 9000), (2000, 20000), (1, 40000), (37, 333)]:
        a, w = a_all[:rows], w_all[:w_rows]
        ax, aw = sq.sq_calibrate_absmax_pair(a, w, norm_gamma=g, eps=1e-6)
        rx = sq.sq_calibrate_absmax(a, norm_gamma=g, eps=1e-6)
        rw = sq.sq_calibrate_absmax(w)
        assert torch.equal(ax, rx) and torch.equal(aw, rw), (rows, w_rows)
    ok_status(sq)


def test_empty_inputs_are_no_ops(sq):
    """No tokens (T = 0) for every activation quantiser and the GEMM, no output channels (N = 0) for the
    weight quantisers: each call returns success without a launch, and the device status stays clean."""
    dev = "cuda"
    K, N = 4096, 264
    fold = torch.ones(K, device=dev)
    x0 = torch.empty(0, K, dtype=torch.bfloat16, device=dev)
    for q, sc in (sq.sq_rmsnorm_smooth_quant(x0, fold), sq.sq_rmsnorm_smooth_quant(x0, fold, apply_norm=False),
                  sq.sq_rmsnorm_smooth_quant_fp8(x0, fold),
                  sq.sq_rmsnorm_smooth_quant_static(x0, fold, sq.sq_static_scale(torch.ones(K, device=dev))),
                  sq.sq_layernorm_smooth_quant(x0, fold, torch.zeros(K, device=dev))):
        assert q.shape == (0, K) and sc.shape == (0,)
    w0 = torch.empty(0, K, dtype=torch.bfloat16, device=dev)
    for wq0, ws0 in (sq.sq_smooth_quantize_weight(w0, fold), sq.sq_smooth_quantize_weight_fp8(w0, fold)):
        assert wq0.shape == (0, K) and ws0.shape == (0,)
    wq = torch.zeros(N, K, dtype=torch.int8, device=dev)
    ws = torch.ones(N, device=dev)
    y = sq.sq_w8a8_linear(torch.empty(0, K, dtype=torch.int8, device=dev), torch.empty(0, device=dev), wq, ws)
    assert y.shape == (0, N)
    ok_status(sq)


# Quantisers over few rows (decode-sized token counts) take one row per group of eight warps, up to 4
# rows per SM; every quantiser mode against the oracle at token counts on both sides of that bound
# (592 rows on 148 SMs), at widths whose rows fill the eight-warp group exactly (4096, 8192) or not
# (2568, 6144).
FEW_ROWS = [(1, 4096), (7, 2568), (64, 8192), (300, 6144), (592, 4096), (593, 4096)]


@pytest.mark.parametrize("T,K", FEW_ROWS)
def test_quantisers_over_few_rows(sq, orc, T, K):
    every_quantiser(sq, orc, T, K, 21)


# The quantisers at the ends of their width range: the narrowest rows (one lane vector, eight rows to a
# warp) and the widest the row kernels hold (16384 elements), full and one vector short of full, at
# token counts that leave a ragged last unit.
WIDTHS = [(1, 8), (333, 8), (3001, 16), (37, 24), (5, 16384), (300, 16384), (129, 16376)]


@pytest.mark.parametrize("T,K", WIDTHS)
def test_quantisers_at_the_width_limits(sq, orc, T, K):
    every_quantiser(sq, orc, T, K, 31)


# Row counts on both sides of the switch between the two unit numberings of the quantisers (group by group
# across the CTAs up to 4 units per row group, CTA by CTA beyond): 4 x 8 groups x 148 SMs = 4736 rows of
# 4096 elements, 4 x 4 x 148 = 2368 rows of 8192.
NUMBERING = [(4736, 4096), (4737, 4096), (2368, 8192), (2369, 8192)]


@pytest.mark.parametrize("T,K", NUMBERING)
def test_quantisers_across_the_unit_numberings(sq, orc, T, K):
    every_quantiser(sq, orc, T, K, 41)


def every_quantiser(sq, orc, T, K, seed):
    """Dynamic INT8 and FP8, static INT8 (with clipping), LayerNorm INT8 and the weight quantiser on
    T rows of K elements, each against the oracle (codes and scales bit-exact)."""
    dev = "cuda"
    ch = synth.outlier_channels(K, synth.OutlierSpec(max(1, K // 256), 10, 40), seed)
    x = synth.outlier_tokens(T, K, ch, seed + 1, dev)
    fold = synth.norm_gamma(K, seed + 2, dev)
    x_h, f_h = h16(x), hnp(fold)
    for norm in (True, False):
        q, sc = sq.sq_rmsnorm_smooth_quant(x, fold, apply_norm=norm)
        rq, rs = orc.rmsnorm_smooth_quant(x_h, f_h, apply_norm=norm)
        assert np.array_equal(hnp(q), rq) and np.array_equal(hnp(sc), rs)
        q, sc = sq.sq_rmsnorm_smooth_quant_fp8(x, fold, apply_norm=norm)
        rq, rs = orc.rmsnorm_smooth_quant_f8(x_h, f_h, apply_norm=norm)
        assert np.array_equal(hnp(q), rq) and np.array_equal(hnp(sc), rs)
    amax_y = np.full(K, 2.0, np.float32)
    amax_y[K // 3] = 6.0                                # values past the calibrated maximum are clipped
    s2 = orc.static_scale(amax_y)
    for norm in (True, False):
        q, sc = sq.sq_rmsnorm_smooth_quant_static(x, fold, torch.from_numpy(s2).to(dev), apply_norm=norm)
        rq, rs = orc.rmsnorm_smooth_quant_static(x_h, f_h, s2, apply_norm=norm)
        assert np.array_equal(hnp(q), rq) and np.array_equal(hnp(sc), rs)
    beta = synth.norm_gamma(K, seed + 3, dev) - 1.0
    q, sc = sq.sq_layernorm_smooth_quant(x + 3, fold, beta)
    rq, rs = orc.layernorm_smooth_quant(h16(x + 3), f_h, hnp(beta))
    assert np.array_equal(hnp(q), rq) and np.array_equal(hnp(sc), rs)
    w = synth.normal_weight(T, K, seed + 4, dev)        # a weight with as few output channels
    q, sc = sq.sq_smooth_quantize_weight(w, fold)
    rq, rs = orc.smooth_quantize_weight(h16(w), f_h)
    assert np.array_equal(hnp(q), rq) and np.array_equal(hnp(sc), rs)
    ok_status(sq)


# The CTA-pair GEMM (cta_group::2, 256 x 256 tiles) against the single-SM form and the oracle:
# ragged T and N, K not a multiple of the 128-byte stage, bias on and off, and T below 256 (which
# keeps the single-SM form even when pairs are enabled).
PAIR_SHAPES = [(256, 256, 128, False), (300, 520, 272, True), (777, 1288, 2064, True), (1024, 4096, 4096, False),
               (200, 264, 512, True)]


@pytest.mark.parametrize("T,N,K,bias", PAIR_SHAPES)
def test_cta_pair_gemm_matches(sq, orc, T, N, K, bias):
    dev = "cuda"
    g = torch.Generator(device="cpu").manual_seed(T + 3 * N + 7 * K)
    xq = torch.randint(-127, 128, (T, K), dtype=torch.int8, generator=g).to(dev)
    wq = torch.randint(-127, 128, (N, K), dtype=torch.int8, generator=g).to(dev)
    xs = (torch.rand(T, generator=g) * 1e-2).to(dev)
    ws = (torch.rand(N, generator=g) * 1e-2).to(dev)
    b = (torch.randn(N, generator=g)).to(torch.bfloat16).to(dev) if bias else None
    outs = []
    try:
        for pair in (False, True):
            sq.sq_set_gemm_cta_pair(pair)
            acc = torch.empty(T, N, dtype=torch.int32, device=dev)
            y = sq.sq_w8a8_linear(xq, xs, wq, ws, bias=b, acc_out=acc)
            ok_status(sq)
            outs.append((y, acc))
    finally:
        sq.sq_set_gemm_cta_pair(False)
    assert torch.equal(outs[0][1], outs[1][1]) and torch.equal(outs[0][0], outs[1][0])
    rows = sample_indices(T, 24, T)
    check_linear(sq, orc, xq, xs, wq, ws, b, outs[1][0], outs[1][1], rows=rows)


# The decode form (weights as the 128-row MMA operand, tokens padded to 16, 32, 64 or 128 columns):
# every padding bucket and its edges, N not a multiple of 128, K not a multiple of the 128-byte stage.
@pytest.mark.parametrize("T", [16, 17, 33, 65, 100, 128])
def test_decode_form_buckets(sq, orc, T):
    dev = "cuda"
    N, K = 1000, 2064
    g = torch.Generator(device="cpu").manual_seed(5 * T)
    xq = torch.randint(-127, 128, (T, K), dtype=torch.int8, generator=g).to(dev)
    wq = torch.randint(-127, 128, (N, K), dtype=torch.int8, generator=g).to(dev)
    xs = (torch.rand(T, generator=g) * 1e-2).to(dev)
    ws = (torch.rand(N, generator=g) * 1e-2).to(dev)
    b = torch.randn(N, generator=g).to(torch.bfloat16).to(dev)
    acc = torch.empty(T, N, dtype=torch.int32, device=dev)
    y = sq.sq_w8a8_linear(xq, xs, wq, ws, bias=b, acc_out=acc)
    ok_status(sq)
    check_linear(sq, orc, xq, xs, wq, ws, b, y, acc)


# Static per-tensor activation scale: the calibration maximum of the quantiser's own y, the per-tensor
# step, and the clipping quantiser, against the oracle fed the same inputs; online tokens include
# values well beyond the calibration range, so saturation is exercised.
@pytest.mark.parametrize("K,norm", [(1024, True), (1040, False), (4096, True), (4096, False), (8192, True)])
def test_static_scale_path(sq, orc, K, norm):
    dev = "cuda"
    Tc, T, N = 1500, 777, 264
    ch = synth.outlier_channels(K, synth.OutlierSpec(max(1, K // 256), 10.0, 25.0), K)
    Xc = synth.outlier_tokens(Tc, K, ch, K + 1, dev)
    X = synth.outlier_tokens(T, K, ch, K + 2, dev)
    W = synth.normal_weight(N, K, K + 3, dev)
    gamma = synth.norm_gamma(K, K + 4, dev) if norm else None
    amax = sq.sq_calibrate_absmax(Xc, norm_gamma=gamma)
    s, fold = sq.sq_compute_scales(amax, sq.sq_calibrate_absmax(W), 0.5, gamma=gamma)
    fold_h = hnp(fold)
    # the first 40 tokens go beyond anything calibration saw, so their codes clip: one channel (the
    # one with the largest fold) dominates each of them (scaling a whole token would not do it with
    # the norm, which is scale free)
    X[:40, int(np.argmax(np.abs(fold_h)))] = 1000.0
    if norm:
        amax_y = sq.sq_calibrate_absmax(Xc, norm_gamma=fold)
        s2 = sq.sq_static_scale(amax_y)
        amax_y_o = orc.calibrate_absmax(h16(Xc), norm_gamma=fold_h)
    else:
        amax_x = sq.sq_calibrate_absmax(Xc)
        s2 = sq.sq_static_scale(amax_x, factor=fold)
        amax_y_o = (orc.calibrate_absmax(h16(Xc)) * np.abs(fold_h)).astype(np.float32)
    ok_status(sq)
    s2_o = orc.static_scale(amax_y_o)
    assert np.array_equal(hnp(s2), s2_o), f"static scale differs: {hnp(s2)} vs {s2_o}"
    xq, xs = sq.sq_rmsnorm_smooth_quant_static(X, fold, s2, apply_norm=norm)
    xq_o, xs_o = orc.rmsnorm_smooth_quant_static(h16(X), fold_h, hnp(s2), apply_norm=norm)
    assert np.array_equal(hnp(xs), xs_o) and np.all(hnp(xs) == hnp(s2)[0])
    assert np.array_equal(hnp(xq), xq_o), f"{int((hnp(xq) != xq_o).sum())} static codes differ"
    assert np.all((np.abs(xq_o[:40]) == 127).sum(axis=1) >= 1)   # every planted token saturates
    wq, ws = sq.sq_smooth_quantize_weight(W, s)
    acc = torch.empty(T, N, dtype=torch.int32, device=dev)
    y = sq.sq_w8a8_linear(xq, xs, wq, ws, acc_out=acc)
    check_linear(sq, orc, xq, xs, wq, ws, None, y, acc)
    ok_status(sq)


# Rows whose maximum m is so small that 127 / m (448 / m for FP8) overflows binary32: the library
# and the oracle both scale such a row by 2^64 before coding it (exact), and with an overflowing static
# reciprocal a zero value codes 0 and every other value saturates. Tiny rows sit next to ordinary rows
# in the same units (one-warp units of several rows, two- and eight-warp row groups), and include a
# row of one subnormal, a zero row and zeros inside tiny rows. Per-token, weight, FP8 and static.
TINY_SHAPES = [(37, 64), (700, 1024), (37, 4096), (700, 4096), (40, 8192)]


def _tiny_rows_dev(T, K, seed):
    rng = np.random.default_rng(seed)
    mag = 2.0 ** rng.uniform(-133, -123, size=(T, K))
    v = (mag * rng.choice([-1.0, 1.0], size=(T, K))).astype(np.float32)
    normal = rng.random(T) < 0.3                       # ordinary rows in between
    normal[:5] = False
    v[normal] = rng.standard_normal((int(normal.sum()), K)).astype(np.float32)
    v[1, :] = 0.0
    v[1, 3] = -2.0 ** -133
    v[2, :] = 0.0
    v[3, 5] = 0.0
    return torch.from_numpy(v).to(torch.bfloat16).cuda()


@pytest.mark.parametrize("T,K", TINY_SHAPES)
def test_tiny_rows_every_quantiser(sq, orc, T, K):
    x = _tiny_rows_dev(T, K, 17 * T + K)
    one = torch.ones(K, dtype=torch.float32, device="cuda")
    xh, oh = h16(x), np.ones(K, np.float32)
    xq, xs = sq.sq_rmsnorm_smooth_quant(x, one, apply_norm=False)
    xq_o, xs_o = orc.rmsnorm_smooth_quant(xh, oh, apply_norm=False)
    assert np.array_equal(hnp(xs), xs_o), "token scales of tiny rows differ"
    assert np.array_equal(hnp(xq), xq_o), f"{int((hnp(xq) != xq_o).sum())} codes of tiny rows differ"
    wq, ws = sq.sq_smooth_quantize_weight(x, None)
    wq_o, ws_o = orc.smooth_quantize_weight(xh)
    assert np.array_equal(hnp(ws), ws_o) and np.array_equal(hnp(wq), wq_o), "weight codes of tiny rows differ"
    fq, fs = sq.sq_rmsnorm_smooth_quant_fp8(x, one, apply_norm=False)
    fq_o, fs_o = orc.rmsnorm_smooth_quant_f8(xh, oh, apply_norm=False)
    assert np.array_equal(hnp(fs), fs_o) and np.array_equal(hnp(fq), fq_o), "fp8 codes of tiny rows differ"
    # a static scale calibrated on tiny values only: 127 / m overflows to +inf
    amax = sq.sq_calibrate_absmax(x[4:5])
    s2 = sq.sq_static_scale(amax)
    s2_o = orc.static_scale(orc.calibrate_absmax(xh[4:5]))
    assert np.array_equal(hnp(s2), s2_o) and np.isinf(s2_o[1])
    sq_q, sq_s = sq.sq_rmsnorm_smooth_quant_static(x, one, s2, apply_norm=False)
    st_o, ss_o = orc.rmsnorm_smooth_quant_static(xh, oh, s2_o, apply_norm=False)
    assert np.array_equal(hnp(sq_s), ss_o) and np.array_equal(hnp(sq_q), st_o), "static codes of tiny rows differ"
    assert np.array_equal(st_o, (np.sign(f64(xh)) * 127).astype(np.int8))
    ok_status(sq)


# Values placed next to the ties k + 1/2 of v * fl32(127/m): the codes round the exact product once
# (a third of these values would move by one code if the product were rounded to binary32 first).
# They enter as the smoothing factors of weight rows of ones, and as the fold of tokens of ones (no
# norm), so y = the designed values exactly; 300 rows reach every row geometry's unit layout.
def test_near_tie_codes_match_the_oracle(sq, orc):
    dev = "cuda"
    m = np.float32(37.123)
    inv = np.float32(127.0) / m
    y = ((np.arange(127) + 0.5) / np.float64(inv)).astype(np.float32)
    row = np.zeros(256, np.float32)
    row[0], row[1:128], row[128:255] = m, y, -y
    for K in (256, 4096):
        f = np.tile(row, K // 256)
        ones = torch.ones(300, K, dtype=torch.bfloat16, device=dev)
        fd = torch.from_numpy(f).to(dev)
        wq, ws = sq.sq_smooth_quantize_weight(ones, fd)
        wq_o, ws_o = orc.smooth_quantize_weight(h16(ones), f)
        assert np.array_equal(hnp(ws), ws_o) and np.array_equal(hnp(wq), wq_o), f"near-tie weight codes differ (K={K})"
        xq, xs = sq.sq_rmsnorm_smooth_quant(ones, fd, apply_norm=False)
        xq_o, xs_o = orc.rmsnorm_smooth_quant(h16(ones), f, apply_norm=False)
        assert np.array_equal(hnp(xs), xs_o) and np.array_equal(hnp(xq), xq_o), f"near-tie token codes differ (K={K})"
        s2 = sq.sq_static_scale(torch.full((K,), float(m), dtype=torch.float32, device=dev))
        sq_q, _ = sq.sq_rmsnorm_smooth_quant_static(ones, fd, s2, apply_norm=False)
        st_o, _ = orc.rmsnorm_smooth_quant_static(h16(ones), f, hnp(s2), apply_norm=False)
        assert np.array_equal(hnp(sq_q), st_o), f"near-tie static codes differ (K={K})"
    ok_status(sq)


# The static quantiser reads the scale that the kernel launched just before it writes (a dependent
# launch: it may start while that kernel still runs). The buffer is refilled with a wrong scale before
# every pair of calls, so a read that does not wait for its producer shows up as wrong codes.
def test_static_scale_read_after_its_producer(sq, orc):
    dev = "cuda"
    T, K = 256, 4096
    ch = synth.outlier_channels(K, synth.OutlierSpec(16, 10.0, 25.0), 5)
    X = synth.outlier_tokens(T, K, ch, 6, dev)
    fold = synth.norm_gamma(K, 7, dev)
    Xh, fh = h16(X), hnp(fold)
    s2 = torch.empty(2, dtype=torch.float32, device=dev)
    for i in range(12):
        amax = (torch.rand(K, device=dev) + 0.5) * (1 + i)
        s2.fill_(1e-30)                                # the wrong scale a stale read would see
        sq.sq_static_scale(amax, scale2=s2)
        xq, xs = sq.sq_rmsnorm_smooth_quant_static(X, fold, s2)
        s2_o = orc.static_scale(hnp(amax))
        xq_o, xs_o = orc.rmsnorm_smooth_quant_static(Xh, fh, s2_o)
        assert np.array_equal(hnp(s2), s2_o)
        assert np.array_equal(hnp(xs), xs_o) and np.array_equal(hnp(xq), xq_o), f"stale static scale at call {i}"
    ok_status(sq)


# Fold into the previous linear layer: bit-exact against the oracle, in place as well; then the
# smoothed layer fed by the folded layer's output quantises with fold = 1 and matches the oracle.
@pytest.mark.parametrize("K,Kp,bias", [(4096, 4096, True), (1000, 264, False), (8, 8, True)])
def test_fold_into_prev_linear(sq, orc, K, Kp, bias):
    dev = "cuda"
    g = torch.Generator(device="cpu").manual_seed(K + Kp)
    w = (torch.randn(K, Kp, generator=g) * 0.05).to(torch.bfloat16).to(dev)
    b = (torch.randn(K, generator=g) * 0.05).to(torch.bfloat16).to(dev) if bias else None
    fold = (0.2 + torch.rand(K, generator=g) * 5).to(dev)
    wo, bo = sq.sq_fold_into_prev_linear(w, fold, b)
    wo_o, bo_o = orc.fold_into_prev_linear(h16(w), h16(b) if bias else None, hnp(fold))
    assert np.array_equal(h16(wo), wo_o)
    if bias:
        assert np.array_equal(h16(bo), bo_o)
    w2, b2 = w.clone(), (b.clone() if bias else None)
    sq.sq_fold_into_prev_linear(w2, fold, b2, w_out=w2, b_out=b2)          # in place
    assert torch.equal(w2, wo) and (not bias or torch.equal(b2, bo))
    ws = torch.rand(K, generator=g).to(dev) * 1e-2
    assert np.array_equal(hnp(sq.sq_fold_into_w_scale(ws, fold)), orc.fold_into_w_scale(hnp(ws), hnp(fold)))
    ok_status(sq)


# FP8 E4M3 variant: codes and scales bit-exact against the oracle; the binary32 tensor-core
# accumulators within the bound of binary32 summation (K * 2^-24 * sum |products|, K the terms) of
# the exact sum; the epilogue bit-exact given those accumulators; the bf16 outputs within the
# 1e-2 bar of the exact dequantised product. Shapes reach every GEMM form (decode, 64- and
# 256-channel tiles) with ragged T, N and K.
FP8_SHAPES = [(1, 264, 144, True, True), (33, 1000, 2064, False, False), (100, 520, 1040, True, True),
              (300, 520, 272, False, True), (2000, 2312, 1040, True, False)]


@pytest.mark.parametrize("T,N,K,norm,bias", FP8_SHAPES)
def test_fp8_path(sq, orc, T, N, K, norm, bias):
    dev = "cuda"
    seed = 3 * T + N + K
    ch = synth.outlier_channels(K, synth.OutlierSpec(max(1, K // 64), 10.0, 100.0), seed)
    X = synth.outlier_tokens(T, K, ch, seed + 1, dev)
    X[T // 2].zero_()
    W = synth.normal_weight(N, K, seed + 2, dev)
    gamma = synth.norm_gamma(K, seed + 3, dev) if norm else None
    b = synth.bias_vector(N, seed + 4, dev) if bias else None
    s, fold = sq.sq_compute_scales(sq.sq_calibrate_absmax(X, norm_gamma=gamma), sq.sq_calibrate_absmax(W), 0.5, gamma=gamma)
    wq, ws = sq.sq_smooth_quantize_weight_fp8(W, s)
    wq_o, ws_o = orc.smooth_quantize_weight_f8(h16(W), hnp(s))
    assert np.array_equal(hnp(ws), ws_o) and np.array_equal(hnp(wq), wq_o), "fp8 weight codes differ"
    xq, xs = sq.sq_rmsnorm_smooth_quant_fp8(X, fold, apply_norm=norm)
    xq_o, xs_o = orc.rmsnorm_smooth_quant_f8(h16(X), hnp(fold), apply_norm=norm)
    assert np.array_equal(hnp(xs), xs_o), "fp8 token scales differ"
    assert np.array_equal(hnp(xq), xq_o), f"{int((hnp(xq) != xq_o).sum())} fp8 token codes differ"
    assert hnp(xs)[T // 2] == 0 and not hnp(xq)[T // 2].any()
    acc = torch.empty(T, N, dtype=torch.float32, device=dev)
    y = sq.sq_w8a8_linear_fp8(xq, xs, wq, ws, bias=b, acc_out=acc)
    ok_status(sq)
    exact = orc.gemm_f8(hnp(xq), hnp(wq))
    table = orc.e4m3_decode(np.arange(256, dtype=np.uint8)).astype(np.float64)
    mag = np.abs(table[hnp(xq)]) @ np.abs(table[hnp(wq)]).T            # sum of |products|, exact
    acc_h = hnp(acc).astype(np.float64)
    assert np.all(np.abs(acc_h - exact) <= K * 2.0 ** -24 * mag + 1e-30), "fp8 accumulators beyond binary32 summation error"
    b_h = h16(b) if bias else None
    assert np.array_equal(h16(y), orc.dequant_f32(hnp(acc), hnp(xs), hnp(ws), b_h)), "fp8 epilogue differs"
    ref = exact * hnp(xs)[:, None].astype(np.float64) * hnp(ws)[None, :] + (f64(b_h)[None, :] if bias else 0.0)
    scale_mag = mag * hnp(xs)[:, None].astype(np.float64) * hnp(ws)[None, :]
    assert np.all(np.abs(f64(h16(y)) - ref) <= 1e-2 * np.abs(ref) + 1e-2 * 2.0 ** -8 * (scale_mag + (np.abs(f64(b_h))[None, :] if bias else 0)) + 1e-30)


# LayerNorm fold: the calibration abs-max of LayerNorm(x) * gamma + beta, the folded bias beta / s and
# the fused LayerNorm + INT8 quantiser, bit-exact against the oracle. Tokens carry a common offset
# (so the centring matters); one row is zero and one constant (both normalise to c = 0, so y is the
# folded bias alone); calibration reads strided rows in two batches (running maximum). Widths reach
# every block shape of the kernel (1, 2 and 4 vectors per thread; 32..512 threads) with ragged ones.
LN_SHAPES = [(300, 64, True), (777, 1040, False), (1000, 4096, True), (513, 8192, True), (129, 12288, False),
             (64, 16384, True)]


@pytest.mark.parametrize("T,K,bias", LN_SHAPES)
def test_layernorm_fold_path(sq, orc, T, K, bias):
    dev = "cuda"
    seed = 7 * T + K
    ch = synth.outlier_channels(K, synth.OutlierSpec(max(1, K // 128), 10.0, 60.0), seed)
    Xc = (synth.outlier_tokens(2 * T, K, ch, seed + 1, dev).float() + 3.0).to(torch.bfloat16)
    X = (synth.outlier_tokens(T, K, ch, seed + 2, dev).float() + 3.0).to(torch.bfloat16)
    X[T // 2].zero_()
    X[T // 3] = 0.75
    g = torch.Generator(device="cpu").manual_seed(seed + 3)
    gamma = (1 + 0.2 * torch.randn(K, generator=g)).to(dev)
    beta = (0.1 * torch.randn(K, generator=g)).to(dev) if bias else None
    zeros = np.zeros(K, np.float32)
    big = torch.zeros(2 * T, K + 16, dtype=torch.bfloat16, device=dev)
    big[:, :K] = Xc
    amax = sq.sq_calibrate_absmax_layernorm(big[:T, :K], gamma, beta)
    sq.sq_calibrate_absmax_layernorm(big[T:, :K], gamma, beta, amax=amax, accumulate=True)
    ok_status(sq)
    amax_o = orc.calibrate_absmax_layernorm(h16(Xc), hnp(gamma), hnp(beta) if bias else zeros)
    assert np.array_equal(hnp(amax), amax_o), f"{int((hnp(amax) != amax_o).sum())} LayerNorm abs-maxima differ"
    N = 264
    W = synth.normal_weight(N, K, seed + 4, dev)
    s, fold = sq.sq_compute_scales(amax, sq.sq_calibrate_absmax(W), 0.5, gamma=gamma)
    bf = sq.sq_fold_layernorm_bias(beta, s) if bias else None
    if bias:
        assert np.array_equal(hnp(bf), orc.fold_layernorm_bias(hnp(beta), hnp(s)))
    xq, xs = sq.sq_layernorm_smooth_quant(X, fold, bf)
    ok_status(sq)
    xq_o, xs_o = orc.layernorm_smooth_quant(h16(X), hnp(fold), hnp(bf) if bias else zeros)
    assert np.array_equal(hnp(xs), xs_o), f"{int((hnp(xs) != xs_o).sum())} LayerNorm token scales differ"
    assert np.array_equal(hnp(xq), xq_o), f"{int((hnp(xq) != xq_o).sum())} LayerNorm codes differ"
    if bias:   # a zero row and a constant row both quantise the folded bias alone
        assert np.array_equal(hnp(xq)[T // 2], hnp(xq)[T // 3]) and hnp(xs)[T // 2] == hnp(xs)[T // 3] > 0
    else:
        assert hnp(xs)[T // 2] == 0 and hnp(xs)[T // 3] == 0 and not hnp(xq)[T // 3].any()
    wq, ws = sq.sq_smooth_quantize_weight(W, s)
    acc = torch.empty(T, N, dtype=torch.int32, device=dev)
    y = sq.sq_w8a8_linear(xq, xs, wq, ws, acc_out=acc)
    check_linear(sq, orc, xq, xs, wq, ws, None, y, acc)
    ok_status(sq)


# Dependent launch: every libsq kernel may start while the previous kernel of the stream finishes, and
# the calibration abs-max reads its rows before its own wait (after the library's zero-fill). Inputs
# written by a long torch kernel immediately before each call (same stream, no synchronisation) must
# be seen complete: results equal those of the same calls on inputs written long before.
def test_inputs_written_just_before_each_call(sq, orc):
    dev = "cuda"
    w = synth.WORKLOADS[1]
    d = synth.group_inputs(w, 0, dev, T=2048)
    gamma, W, X = d["gamma"], d["weight"], d["x"]
    calib = torch.cat(list(synth.calibration_chunks(w, d["channels"], dev)))[:16384]
    ref_amax = sq.sq_calibrate_absmax(calib, norm_gamma=gamma)
    ref_aw = sq.sq_calibrate_absmax(W)
    ref_s, ref_fold = sq.sq_compute_scales(ref_amax, ref_aw, 0.5, gamma=gamma)
    ref_wq, ref_ws = sq.sq_smooth_quantize_weight(W, ref_s)
    ref_xq, ref_xs = sq.sq_rmsnorm_smooth_quant(X, ref_fold)
    ref_y = sq.sq_w8a8_linear(ref_xq, ref_xs, ref_wq, ref_ws)
    torch.cuda.synchronize()
    big = torch.empty(256 * 1024 * 1024 // 2, dtype=torch.bfloat16, device=dev)   # 256 MB: a kernel of ~100 us
    for trial in range(3):
        c2, W2, X2 = torch.empty_like(calib), torch.empty_like(W), torch.empty_like(X)
        torch.cuda.synchronize()
        big.fill_(trial)                      # keeps the stream busy, then the input is written last
        c2.copy_(calib)
        amax = sq.sq_calibrate_absmax(c2, norm_gamma=gamma)
        big.fill_(trial + 1)
        W2.copy_(W)
        aw = sq.sq_calibrate_absmax(W2)
        s, fold = sq.sq_compute_scales(amax, aw, 0.5, gamma=gamma)
        wq, ws = sq.sq_smooth_quantize_weight(W2, s)
        big.fill_(trial + 2)
        X2.copy_(X)
        xq, xs = sq.sq_rmsnorm_smooth_quant(X2, fold)
        y = sq.sq_w8a8_linear(xq, xs, wq, ws)
        ok_status(sq)
        assert torch.equal(amax, ref_amax) and torch.equal(aw, ref_aw)
        assert torch.equal(s, ref_s) and torch.equal(fold, ref_fold)
        assert torch.equal(wq, ref_wq) and torch.equal(ws, ref_ws)
        assert torch.equal(xq, ref_xq) and torch.equal(xs, ref_xs) and torch.equal(y, ref_y)
    # and the reference chain itself against the oracle on its calibration maximum
    assert np.array_equal(hnp(ref_amax), orc.calibrate_absmax(h16(calib), norm_gamma=hnp(gamma), eps=1e-6))


# The online path captured in a CUDA graph (its launches carry the dependent-launch attribute) replays
# to the same bits as eager calls, for new input values copied into the captured buffers.
def test_online_path_in_cuda_graph(sq):
    dev = "cuda"
    w = synth.WORKLOADS[1]
    d = synth.group_inputs(w, 0, dev, T=1024)
    gamma, W, X = d["gamma"], d["weight"], d["x"]
    s, fold = sq.sq_compute_scales(sq.sq_calibrate_absmax(X, norm_gamma=gamma), sq.sq_calibrate_absmax(W), 0.5,
                                   gamma=gamma)
    wq, ws = sq.sq_smooth_quantize_weight(W, s)
    xin = X.clone()
    xq = torch.empty(X.shape, dtype=torch.int8, device=dev)
    xs = torch.empty(X.shape[0], dtype=torch.float32, device=dev)
    y = torch.empty(X.shape[0], W.shape[0], dtype=torch.bfloat16, device=dev)

    def online():
        sq.sq_rmsnorm_smooth_quant(xin, fold, xq=xq, x_scale=xs)
        sq.sq_w8a8_linear(xq, xs, wq, ws, y=y)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        online()                                   # warm-up: one-time launch configuration
    torch.cuda.current_stream().wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        online()
    for k in range(3):
        xnew = (X.float() * (1.0 + 0.25 * k) + 0.01 * k).to(torch.bfloat16)
        xin.copy_(xnew)
        graph.replay()
        torch.cuda.synchronize()
        y_graph = y.clone()
        xq_e, xs_e = sq.sq_rmsnorm_smooth_quant(xnew, fold)
        y_e = sq.sq_w8a8_linear(xq_e, xs_e, wq, ws)
        ok_status(sq)
        assert torch.equal(xq, xq_e) and torch.equal(xs, xs_e) and torch.equal(y_graph, y_e)


def test_offline_path_in_cuda_graph(sq):
    """The offline steps (the abs-max pair after its zero-fill, the scales, the weight quantiser)
    captured once in a CUDA graph and replayed on new calibration rows and weights: every output equals
    the one of direct calls."""
    dev = "cuda"
    w = synth.WORKLOADS[1]
    d = synth.group_inputs(w, 0, dev, T=2048)
    gamma, W0, X0 = d["gamma"], d["weight"], d["x"]
    cal, wt = X0.clone(), W0.clone()
    K, N = W0.shape[1], W0.shape[0]
    amax = torch.empty(K, device=dev)
    aw = torch.empty(K, device=dev)
    s = torch.empty(K, device=dev)
    fold = torch.empty(K, device=dev)
    wq = torch.empty(N, K, dtype=torch.int8, device=dev)
    ws = torch.empty(N, device=dev)

    def offline():
        sq.sq_calibrate_absmax_pair(cal, wt, norm_gamma=gamma, amax=amax, amax_w=aw)
        sq.sq_compute_scales(amax, aw, 0.5, gamma=gamma, s=s, fold=fold)
        sq.sq_smooth_quantize_weight(wt, s, wq=wq, w_scale=ws)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        offline()                                  # warm-up: one-time launch configuration
    torch.cuda.current_stream().wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        offline()
    for k in range(3):
        cnew = (X0.float() * (1.0 + 0.5 * k) + 0.02 * k).to(torch.bfloat16)
        wnew = (W0.float() * (1.0 - 0.2 * k)).to(torch.bfloat16)
        cal.copy_(cnew)
        wt.copy_(wnew)
        graph.replay()
        torch.cuda.synchronize()
        ax_e, aw_e = sq.sq_calibrate_absmax_pair(cnew, wnew, norm_gamma=gamma)
        s_e, f_e = sq.sq_compute_scales(ax_e, aw_e, 0.5, gamma=gamma)
        wq_e, ws_e = sq.sq_smooth_quantize_weight(wnew, s_e)
        ok_status(sq)
        assert torch.equal(amax, ax_e) and torch.equal(aw, aw_e)
        assert torch.equal(s, s_e) and torch.equal(fold, f_e)
        assert torch.equal(wq, wq_e) and torch.equal(ws, ws_e)


# The variant rows at the query-projection size (T 8192, K = N 4096, the calibration set of 65536 rows), in
# the launch configuration the bench uses for the INT8 path: every code and scale compared with the
# oracle; the GEMMs on sampled full rows and full columns (INT8: bit-exact; FP8: binary32 summation bound,
# epilogue bit-exact).
def test_variants_at_query_projection_size(sq, orc):
    dev = "cuda"
    w = synth.WORKLOADS[1]
    d = synth.group_inputs(w, 0, dev)
    gamma, W, X = d["gamma"], d["weight"], d["x"]
    T, K, N = X.shape[0], X.shape[1], W.shape[0]
    chunks = list(synth.calibration_chunks(w, d["channels"], dev))
    rows = sample_indices(T, 24, 91)
    cols = sample_indices(N, 24, 92)
    amax = torch.empty(K, dtype=torch.float32, device=dev)
    for i, c in enumerate(chunks):
        sq.sq_calibrate_absmax(c, norm_gamma=gamma, eps=w.eps, amax=amax, accumulate=i > 0)
    s, fold = sq.sq_compute_scales(amax, sq.sq_calibrate_absmax(W), 0.5, gamma=gamma)
    s_h, fold_h = hnp(s), hnp(fold)
    x16 = h16(X)
    # f2: static per-tensor scale
    amax_y = torch.empty(K, dtype=torch.float32, device=dev)
    for i, c in enumerate(chunks):
        sq.sq_calibrate_absmax(c, norm_gamma=fold, eps=w.eps, amax=amax_y, accumulate=i > 0)
    s2 = sq.sq_static_scale(amax_y)
    assert np.array_equal(hnp(s2), orc.static_scale(hnp(amax_y)))
    xq, xs = sq.sq_rmsnorm_smooth_quant_static(X, fold, s2, eps=w.eps)
    xq_o, xs_o = orc.rmsnorm_smooth_quant_static(x16, fold_h, hnp(s2), eps=w.eps)
    assert np.array_equal(hnp(xq), xq_o) and np.array_equal(hnp(xs), xs_o)
    wq, ws = sq.sq_smooth_quantize_weight(W, s)
    acc = torch.empty(T, N, dtype=torch.int32, device=dev)
    y = sq.sq_w8a8_linear(xq, xs, wq, ws, acc_out=acc)
    check_linear(sq, orc, xq, xs, wq, ws, None, y, acc, rows=rows, cols=None)
    check_linear(sq, orc, xq, xs, wq, ws, None, y, acc, rows=None, cols=cols)
    # f3: FP8 E4M3
    wq8, ws8 = sq.sq_smooth_quantize_weight_fp8(W, s)
    wq8_o, ws8_o = orc.smooth_quantize_weight_f8(h16(W), s_h)
    assert np.array_equal(hnp(wq8), wq8_o) and np.array_equal(hnp(ws8), ws8_o)
    xq8, xs8 = sq.sq_rmsnorm_smooth_quant_fp8(X, fold, eps=w.eps)
    xq8_o, xs8_o = orc.rmsnorm_smooth_quant_f8(x16, fold_h, eps=w.eps)
    assert np.array_equal(hnp(xq8), xq8_o) and np.array_equal(hnp(xs8), xs8_o)
    accf = torch.empty(T, N, dtype=torch.float32, device=dev)
    y8 = sq.sq_w8a8_linear_fp8(xq8, xs8, wq8, ws8, acc_out=accf)
    ok_status(sq)
    table = orc.e4m3_decode(np.arange(256, dtype=np.uint8)).astype(np.float64)
    for rr, cc in ((rows, None), (None, cols)):
        exact = orc.gemm_f8(hnp(xq8), hnp(wq8), rr, cc)
        xa = np.abs(table[hnp(xq8)[rr] if rr is not None else hnp(xq8)])
        wa = np.abs(table[hnp(wq8)[cc] if cc is not None else hnp(wq8)])
        mag = xa @ wa.T
        a_g = hnp(accf)
        a_g = a_g[rr] if rr is not None else a_g[:, cc]
        assert np.all(np.abs(a_g.astype(np.float64) - exact) <= K * 2.0 ** -24 * mag + 1e-30)
        y_g = h16(y8)
        y_g = y_g[rr] if rr is not None else y_g[:, cc]
        assert np.array_equal(y_g, orc.dequant_f32(np.ascontiguousarray(a_g), hnp(xs8), hnp(ws8), None, rr, cc))
    # f4 (b): LayerNorm fold (gamma reused as the LayerNorm scale, a seeded beta)
    beta = (0.05 * torch.randn(K, generator=torch.Generator(device="cpu").manual_seed(93))).to(dev)
    amax_ln = torch.empty(K, dtype=torch.float32, device=dev)
    amax_ln_o = np.zeros(K, np.float32)
    for i, c in enumerate(chunks):
        sq.sq_calibrate_absmax_layernorm(c, gamma, beta, amax=amax_ln, accumulate=i > 0)
        orc.calibrate_absmax_layernorm(h16(c), hnp(gamma), hnp(beta), amax=amax_ln_o, accumulate=i > 0)
    ok_status(sq)
    assert np.array_equal(hnp(amax_ln), amax_ln_o)
    s_ln, fold_ln = sq.sq_compute_scales(amax_ln, sq.sq_calibrate_absmax(W), 0.5, gamma=gamma)
    bf = sq.sq_fold_layernorm_bias(beta, s_ln)
    assert np.array_equal(hnp(bf), orc.fold_layernorm_bias(hnp(beta), hnp(s_ln)))
    xq_ln, xs_ln = sq.sq_layernorm_smooth_quant(X, fold_ln, bf)
    xq_ln_o, xs_ln_o = orc.layernorm_smooth_quant(x16, hnp(fold_ln), hnp(bf))
    assert np.array_equal(hnp(xq_ln), xq_ln_o) and np.array_equal(hnp(xs_ln), xs_ln_o)
    wq_ln, ws_ln = sq.sq_smooth_quantize_weight(W, s_ln)
    y_ln = sq.sq_w8a8_linear(xq_ln, xs_ln, wq_ln, ws_ln, acc_out=acc)
    check_linear(sq, orc, xq_ln, xs_ln, wq_ln, ws_ln, None, y_ln, acc, rows=rows, cols=None)
    check_linear(sq, orc, xq_ln, xs_ln, wq_ln, ws_ln, None, y_ln, acc, rows=None, cols=cols)
    ok_status(sq)


# Calls from several host threads at once, each on its own stream (the launch configuration caches
# are shared between threads): every thread gets the bits the same calls give one after another.
def test_concurrent_host_threads(sq):
    import threading
    dev = "cuda"
    shapes = [(300, 1032, 2064), (129, 2056, 1040), (1000, 520, 4096), (64, 3000, 272)]
    inputs = []
    for i, (T, N, K) in enumerate(shapes):
        g = torch.Generator(device="cpu").manual_seed(500 + i)
        X = torch.randn(T, K, generator=g).to(torch.bfloat16).to(dev)
        W = (torch.randn(N, K, generator=g) * 0.02).to(torch.bfloat16).to(dev)
        gamma = (1 + 0.1 * torch.randn(K, generator=g)).to(dev)
        inputs.append((X, W, gamma))

    def chain(X, W, gamma, stream):
        with torch.cuda.stream(stream):
            s, fold = sq.sq_compute_scales(sq.sq_calibrate_absmax(X, norm_gamma=gamma), sq.sq_calibrate_absmax(W), 0.5,
                                           gamma=gamma)
            wq, ws = sq.sq_smooth_quantize_weight(W, s)
            xq, xs = sq.sq_rmsnorm_smooth_quant(X, fold)
            return sq.sq_w8a8_linear(xq, xs, wq, ws)

    ref = [chain(*inp, torch.cuda.current_stream()) for inp in inputs]
    torch.cuda.synchronize()
    for _ in range(3):
        out = [None] * len(inputs)
        streams = [torch.cuda.Stream() for _ in inputs]
        errors = []

        def work(i):
            try:
                out[i] = chain(*inputs[i], streams[i])
            except Exception as e:           # reported below, in the main thread
                errors.append(e)

        threads = [threading.Thread(target=work, args=(i,)) for i in range(len(inputs))]
        for t in threads:
            t.start()
        for t in threads:
            t.join()
        torch.cuda.synchronize()
        assert not errors, errors
        ok_status(sq)
        for a, b in zip(out, ref):
            assert torch.equal(a, b)


# The decode form in a chain of calls on distinct weights, each call's tokens and scales written by a
# torch kernel right before it on the same stream: bits equal to the same calls on inputs written
# long before, and to the oracle.
@pytest.mark.parametrize("T", [1, 17, 64, 128])
def test_decode_chain_inputs_written_just_before(sq, orc, T):
    dev = "cuda"
    N, K, L = 2056, 4096, 4
    g = torch.Generator(device="cpu").manual_seed(900 + T)
    ws_ = [(torch.randint(-127, 128, (N, K), generator=g, dtype=torch.int8).to(dev), (torch.rand(N, generator=g) * 1e-2).to(dev))
           for _ in range(L)]
    xq_src = torch.randint(-127, 128, (T, K), generator=g, dtype=torch.int8).to(dev)
    xs_src = (torch.rand(T, generator=g) * 1e-2).to(dev)
    b = (torch.randn(N, generator=g) * 0.1).to(torch.bfloat16).to(dev)
    ref = []
    for wq, wsc in ws_:
        acc = torch.empty(T, N, dtype=torch.int32, device=dev)
        ref.append((sq.sq_w8a8_linear(xq_src, xs_src, wq, wsc, bias=b, acc_out=acc), acc))
    torch.cuda.synchronize()
    for _ in range(3):
        got = []
        for wq, wsc in ws_:
            xq, xs = torch.empty_like(xq_src), torch.empty_like(xs_src)
            xq.copy_(xq_src)
            xs.copy_(xs_src)
            acc = torch.empty(T, N, dtype=torch.int32, device=dev)
            got.append((sq.sq_w8a8_linear(xq, xs, wq, wsc, bias=b, acc_out=acc), acc))
        torch.cuda.synchronize()
        ok_status(sq)
        for (y, acc), (y0, acc0) in zip(got, ref):
            assert torch.equal(acc, acc0) and torch.equal(y, y0)
    check_linear(sq, orc, xq_src, xs_src, ws_[0][0], ws_[0][1], b, ref[0][0], ref[0][1])


# The user-facing layer object (SmoothedW8A8Linear): calibrate on batches, then forward, for every norm
# / scheme it offers, against the oracle chain fed the layer's own s and fold (codes, scales and bf16
# outputs bit-exact; FP8 accumulators within the binary32 summation bound).
LAYER_CASES = [("rms", "int8"), ("rms", "int8_static"), ("rms", "fp8"), ("none", "int8"), ("none", "int8_static"),
               ("none", "fp8"), ("layer", "int8")]


@pytest.mark.parametrize("norm,scheme", LAYER_CASES)
def test_layer_object(sq, orc, norm, scheme):
    from post_quantization_calib_b200.layer import SmoothedW8A8Linear
    dev = "cuda"
    T, K, Ns = 300, 1040, (264, 256)
    seed = 70 + LAYER_CASES.index((norm, scheme))
    ch = synth.outlier_channels(K, synth.OutlierSpec(12, 10.0, 40.0), seed)
    batches = [synth.outlier_tokens(200, K, ch, seed + 1 + i, dev) for i in range(3)]
    x = synth.outlier_tokens(T, K, ch, seed + 9, dev)
    ws = [synth.normal_weight(n, K, seed + 10 + i, dev) for i, n in enumerate(Ns)]
    g = torch.Generator(device="cpu").manual_seed(seed)
    gamma = (1 + 0.1 * torch.randn(K, generator=g)).to(dev) if norm != "none" else None
    beta = (0.05 * torch.randn(K, generator=g)).to(dev) if norm == "layer" else None
    bias = synth.bias_vector(sum(Ns), seed + 20, dev)
    layer = SmoothedW8A8Linear(ws, 0.5, gamma=gamma, beta=beta, bias=bias, norm=None if norm == "none" else norm,
                               scheme=scheme)
    layer.calibrate(batches)
    N = layer.N
    acc = torch.empty(T, N, dtype=torch.float32 if scheme == "fp8" else torch.int32, device=dev)
    y = layer(x, acc_out=acc)
    ok_status(sq)
    cal = np.concatenate([h16(b) for b in batches])
    g_h = hnp(gamma) if gamma is not None else None
    if norm == "layer":
        amax_o = orc.calibrate_absmax_layernorm(cal, g_h, hnp(beta), eps=layer.eps)
    else:
        amax_o = orc.calibrate_absmax(cal, norm_gamma=g_h, eps=layer.eps)
    assert np.array_equal(hnp(layer.amax_x), amax_o)
    s_o, _ = orc.compute_scales(amax_o, orc.calibrate_absmax(h16(layer.weight)), 0.5, g_h)
    assert np.all(np.abs(hnp(layer.s).astype(np.float64) / s_o - 1) <= 1e-6)
    s_h, f_h, x16 = hnp(layer.s), hnp(layer.fold), h16(x)
    if scheme == "fp8":
        wq_o, ws_o = orc.smooth_quantize_weight_f8(h16(layer.weight), s_h)
        xq_o, xs_o = orc.rmsnorm_smooth_quant_f8(x16, f_h, eps=layer.eps, apply_norm=norm == "rms")
    else:
        wq_o, ws_o = orc.smooth_quantize_weight(h16(layer.weight), s_h)
        if norm == "layer":
            bf_o = orc.fold_layernorm_bias(hnp(beta), s_h)
            assert np.array_equal(hnp(layer.beta_fold), bf_o)
            xq_o, xs_o = orc.layernorm_smooth_quant(x16, f_h, bf_o, eps=layer.eps)
        elif scheme == "int8_static":
            if norm == "rms":
                amax_y = orc.calibrate_absmax(cal, norm_gamma=f_h, eps=layer.eps)
            else:
                amax_y = (orc.calibrate_absmax(cal) * np.abs(f_h)).astype(np.float32)
            s2_o = orc.static_scale(amax_y)
            assert np.array_equal(hnp(layer.scale2), s2_o)
            xq_o, xs_o = orc.rmsnorm_smooth_quant_static(x16, f_h, s2_o, eps=layer.eps, apply_norm=norm == "rms")
        else:
            xq_o, xs_o = orc.rmsnorm_smooth_quant(x16, f_h, eps=layer.eps, apply_norm=norm == "rms")
    assert np.array_equal(hnp(layer.wq), wq_o) and np.array_equal(hnp(layer.w_scale), ws_o)
    if scheme == "fp8":
        exact = orc.gemm_f8(xq_o, wq_o)
        table = orc.e4m3_decode(np.arange(256, dtype=np.uint8)).astype(np.float64)
        mag = np.abs(table[xq_o]) @ np.abs(table[wq_o]).T
        assert np.all(np.abs(hnp(acc).astype(np.float64) - exact) <= K * 2.0 ** -24 * mag + 1e-30)
        assert np.array_equal(h16(y), orc.dequant_f32(hnp(acc), xs_o, ws_o, h16(bias)))
    else:
        y_o, acc_o = orc.w8a8_linear(xq_o, xs_o, wq_o, ws_o, h16(bias))
        assert np.array_equal(hnp(acc), acc_o) and np.array_equal(h16(y), y_o)
    assert [t.shape[1] for t in layer.split_output(y)] == list(Ns)


# Layer object, input used directly: 1/s folded into the previous linear layer (bf16 weight and bias,
# in place, bit-exact against the oracle fold); the layer then quantises with factor 1, and its output
# on the folded previous layer's output stays within quantisation error of the unfolded path.
def test_layer_fold_into_previous(sq, orc):
    from post_quantization_calib_b200.layer import SmoothedW8A8Linear
    dev = "cuda"
    T, Kp, K, N = 256, 512, 1024, 264
    g = torch.Generator(device="cpu").manual_seed(81)
    w_prev = (torch.randn(K, Kp, generator=g) * 0.05).to(torch.bfloat16).to(dev)
    b_prev = (torch.randn(K, generator=g) * 0.05).to(torch.bfloat16).to(dev)
    x_in = torch.randn(T, Kp, generator=g).to(torch.bfloat16).to(dev)
    W = synth.normal_weight(N, K, 82, dev)
    h = torch.nn.functional.linear(x_in, w_prev, b_prev)          # the previous layer, run by the caller
    layer = SmoothedW8A8Linear([W], 0.5, scheme="int8")
    layer.calibrate([h])
    y_unfolded = layer(h)
    fold = layer.fold.clone()
    w_o, b_o = orc.fold_into_prev_linear(h16(w_prev), h16(b_prev), hnp(fold))
    layer.fold_into_previous(w_prev, b_prev)
    assert np.array_equal(h16(w_prev), w_o) and np.array_equal(h16(b_prev), b_o)
    assert torch.equal(layer.fold, torch.ones_like(layer.fold))
    h2 = torch.nn.functional.linear(x_in, w_prev, b_prev)          # arrives already divided by s
    y_folded = layer(h2)
    ok_status(sq)
    ref = h.double() @ W.double().t()
    err_u = torch.linalg.vector_norm(y_unfolded.double() - ref) / torch.linalg.vector_norm(ref)
    err_f = torch.linalg.vector_norm(y_folded.double() - ref) / torch.linalg.vector_norm(ref)
    assert err_f < 1.5 * err_u + 1e-3, (float(err_u), float(err_f))


def test_deterministic_bytes(sq):
    w = synth.WORKLOADS[1]
    d = synth.group_inputs(w, 0, "cuda", T=1000)
    amax = sq.sq_calibrate_absmax(d["x"], norm_gamma=d["gamma"])
    aw = sq.sq_calibrate_absmax(d["weight"])
    s, fold = sq.sq_compute_scales(amax, aw, 0.5, gamma=d["gamma"])
    wq, ws = sq.sq_smooth_quantize_weight(d["weight"], s)
    outs = []
    for _ in range(2):
        xq, xs = sq.sq_rmsnorm_smooth_quant(d["x"], fold)
        y = sq.sq_w8a8_linear(xq, xs, wq, ws)
        outs.append((xq.clone(), xs.clone(), y.clone(), sq.sq_calibrate_absmax(d["x"], norm_gamma=d["gamma"]).clone()))
    for a, b in zip(*outs):
        assert torch.equal(a, b)


def test_misaligned_device_pointer_rejected(sq):
    dev = "cuda"
    buf = torch.zeros(64 * 64 + 8, dtype=torch.int8, device=dev)
    xq = buf[1:1 + 64 * 64].view(64, 64)          # 1-byte offset
    wq = torch.zeros(64, 64, dtype=torch.int8, device=dev)
    with pytest.raises(sq.SQError) as e:
        sq.sq_w8a8_linear(xq, torch.ones(64, device=dev), wq, torch.ones(64, device=dev))
    assert e.value.status == 3


def test_bounded_wait_times_out_and_context_survives(sq):
    sq.sq_set_wait_timeout_ns(2_000_000)           # 2 ms
    try:
        sq.sq_selftest_wait_timeout()
        assert sq.sq_device_status() == 6          # SQ_ERR_TIMEOUT, recorded by the kernel
        assert sq.sq_device_status() == 0          # reading cleared it
    finally:
        sq.sq_set_wait_timeout_ns(2_000_000_000)
    # the context is still usable: a normal GEMM runs and reports no error
    xq = torch.ones(128, 256, dtype=torch.int8, device="cuda")
    y = sq.sq_w8a8_linear(xq, torch.ones(128, device="cuda"), xq.clone(), torch.ones(128, device="cuda"))
    assert sq.sq_device_status() == 0
    assert torch.all(y.float() == 256.0)
