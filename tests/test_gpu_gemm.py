"""GPU parity of nvfp4_gemm against the oracle: every FP32 output within
1e-5 * sum_k |a_k w_k| of the float64 product of the exactly decoded operands
(the tolerance of the benchmark spec), outputs with a zero bound exactly 0; the
fused GELU + NVFP4 requantization epilogue checked step by step."""
import numpy as np
import pytest
import torch

import nvfp4_w4a4_quantized_amax_b200 as nv
import oracle
import synth
from gpu_helpers import canonical, dev_bf16, device_status, gpu_quantize, host_bits

pytestmark = pytest.mark.gpu

TOL = 1e-5


def gemm_case(a_bits, w_bits, out_bf16=False, rows=None):
    qa, _ = gpu_quantize(a_bits, nv.SF_MMA)
    qw, _ = gpu_quantize(w_bits, nv.SF_MMA)
    M, N = a_bits.shape[0], w_bits.shape[0]
    c = torch.full((M, N), float("nan"), dtype=torch.bfloat16 if out_bf16 else torch.float32,
                   device="cuda")
    nv.nvfp4_gemm(qa, qw, c)
    torch.cuda.synchronize()
    ac, asc, ag = canonical(qa)
    wc, wsc, wg = canonical(qw)
    ref, bound = oracle.gemm_ref(ac, asc, ag, wc, wsc, wg, rows=rows)
    got = c.float().cpu().numpy().astype(np.float64)
    if rows is not None:
        got = got[rows]
    return got, ref, bound, (qa, qw)


def assert_within_bound(got, ref, bound, extra_rel=0.0):
    err = np.abs(got - ref)
    lim = TOL * bound + extra_rel * np.abs(ref)
    bad = np.argwhere(err > lim)
    assert bad.size == 0, (f"{len(bad)} outputs outside the bound; worst ratio "
                           f"{float(np.max(err / np.maximum(bound, 1e-300))):.3e}")
    zero = bound == 0
    assert np.all(got[zero] == 0)


def test_tiny_linear_128x256x512(cuda_dev):
    a, w = synth.tiny_linear(0)
    got, ref, bound, _ = gemm_case(a, w)
    assert_within_bound(got, ref, bound)
    assert device_status() == nv.OK


@pytest.mark.parametrize("M,N,K", [(1, 16, 16), (300, 272, 400), (129, 144, 1040), (64, 512, 3072),
                                   (513, 256, 256)])
def test_ragged_shapes(cuda_dev, M, N, K):
    a = synth.activations(21, M, K)
    w = synth.weights(21, 0, N, K)
    got, ref, bound, _ = gemm_case(a, w)
    assert_within_bound(got, ref, bound)


def test_bf16_output(cuda_dev):
    a = synth.activations(22, 200, 512)
    w = synth.weights(22, 0, 384, 512)
    got, ref, bound, _ = gemm_case(a, w, out_bf16=True)
    # the bf16 store adds one rounding of the FP32 result (half an ulp at 8 bits)
    assert_within_bound(got, ref, bound, extra_rel=2.0 ** -8)


def test_zero_rows_and_columns_are_exact(cuda_dev):
    a = synth.activations(23, 130, 256)
    w = synth.weights(23, 0, 160, 256)
    a[5] = 0
    w[17] = 0x8000
    got, ref, bound, _ = gemm_case(a, w)
    assert np.all(got[5] == 0) and np.all(got[:, 17] == 0)
    assert_within_bound(got, ref, bound)


@pytest.mark.parametrize("M,N", [(256, 512), (128, 256)])  # CTA-pair kernel, single-CTA kernel
def test_fused_epilogue_nonfinite_blocks(cuda_dev, M, N):
    """A tensor scale of A large enough to overflow part of c: GELU(+inf) = +inf and
    GELU(-inf) = -inf * 0 = NaN.  A 16-block of h holding a NaN gets the E4M3 NaN scale
    0x7F and codes that keep only the signs; a block with infinities and no NaN
    saturates to scale 448 (0x7E) with code 7 (+6) for +inf; every finite block is the
    oracle's quantization of the GPU's h; the reported max|h| is NaN, so an amax
    history rejects it."""
    K = 256
    qx, _ = gpu_quantize(synth.activations(31, M, K), nv.SF_MMA)
    qw, _ = gpu_quantize(synth.weights(31, 0, N, K), nv.SF_MMA)
    c = torch.empty((M, N), dtype=torch.float32, device="cuda")
    nv.nvfp4_gemm(qx, qw, c)
    cmax = float(c.abs().max())
    qx.gscale.mul_(float(np.float32(3.0e38 / (0.6 * cmax))))  # |c| above ~0.7 max overflows
    h = torch.empty((M, N), dtype=torch.float32, device="cuda")
    nv.nvfp4_gemm(qx, qw, None, act=nv.ACT_GELU_TANH, h_out=h)
    hn = h.cpu().numpy()
    fin = np.isfinite(hn)
    assert np.isnan(hn).any() and np.isposinf(hn).any() and fin.mean() > 0.5
    g_h = np.float32(np.abs(hn[fin]).max() / np.float32(2688.0))
    q_h = nv.NVFP4Tensor(M, N, nv.SF_MMA)
    amax = torch.zeros(1, dtype=torch.float32, device="cuda")
    h2 = torch.empty((M, N), dtype=torch.float32, device="cuda")
    nv.nvfp4_gemm(qx, qw, None, act=nv.ACT_GELU_TANH, q_out=q_h,
                  q_gscale_in=torch.tensor([g_h], dtype=torch.float32, device="cuda"),
                  q_amax_out=amax, h_out=h2)
    torch.cuda.synchronize()
    assert device_status() == nv.OK
    assert np.array_equal(h2.cpu().numpy(), hn, equal_nan=True)
    assert np.isnan(amax.item())
    codes, scales, g = canonical(q_h)
    blocks = hn.reshape(M, N // 16, 16)
    nan_b = np.isnan(blocks).any(axis=2)
    inf_b = np.isinf(blocks).any(axis=2) & ~nan_b
    fin_b = ~(nan_b | inf_b)
    assert nan_b.any() and inf_b.any() and fin_b.any()
    assert np.all(scales[nan_b] == 0x7F)
    assert np.all(scales[inf_b] == 0x7E)
    nib = np.stack([codes & 0xF, codes >> 4], axis=-1).reshape(M, N)
    in_inf_b = np.repeat(inf_b, 16, axis=1)
    assert np.all(nib[np.isposinf(hn) & in_inf_b] == 0x7)
    assert np.all(nib[np.repeat(nan_b, 16, axis=1)] & 0x7 == 0)  # NaN blocks: signs only
    hz = np.where(np.repeat(fin_b, 16, axis=1), hn, np.float32(0)).astype(np.float32)
    ref = oracle.quantize(hz, gscale=float(g_h))
    assert np.array_equal(scales[fin_b], ref.scales[fin_b])
    fin_bytes = np.repeat(fin_b, 8, axis=1)
    assert np.array_equal(codes[fin_bytes], ref.codes[fin_bytes])


@pytest.mark.slow
@pytest.mark.parametrize("K,N", [(3072, 3072), (3072, 9216), (3072, 14336), (14336, 3072)])
def test_full_size_block_gemms_sampled_rows(cuda_dev, K, N):
    """M = 8192 tokens: activations 0.5 * t3 with picked channels x30, weights
    N(0, 0.02).  Rows sampled across every 128-row tile, all N columns each."""
    a = synth.activations(2, 8192, K)
    w = synth.weights(2, {3072: 0, 9216: 1, 14336: 2}[N] if K == 3072 else 3, N, K)
    rows = np.unique(np.concatenate([np.arange(0, 8192, 97), [8191]]))
    got, ref, bound, _ = gemm_case(a, w, rows=rows)
    assert_within_bound(got, ref, bound)


def fused_case(M, N, K, seed):
    x = synth.activations(seed, M, K)
    w1 = synth.weights(seed, 0, N, K)
    qx, _ = gpu_quantize(x, nv.SF_MMA)
    qw, _ = gpu_quantize(w1, nv.SF_MMA)
    # plain GEMM: the FP32 pre-activation c
    c = torch.empty((M, N), dtype=torch.float32, device="cuda")
    nv.nvfp4_gemm(qx, qw, c)
    # calibration call: max|h| of this very input gives the supplied scale
    amax = torch.zeros(1, dtype=torch.float32, device="cuda")
    h = torch.empty((M, N), dtype=torch.float32, device="cuda")
    nv.nvfp4_gemm(qx, qw, None, act=nv.ACT_GELU_TANH, h_out=h, q_amax_out=amax)
    g_h = np.float32(amax.item()) / np.float32(2688.0)
    q_h = nv.NVFP4Tensor(M, N, nv.SF_MMA)
    q_h.scales.fill_(0x7F)  # padding must be overwritten with zeros
    gin = torch.tensor([g_h], dtype=torch.float32, device="cuda")
    amax2 = torch.zeros(1, dtype=torch.float32, device="cuda")
    h2 = torch.empty((M, N), dtype=torch.float32, device="cuda")
    nv.nvfp4_gemm(qx, qw, None, act=nv.ACT_GELU_TANH, q_out=q_h, q_gscale_in=gin,
                  q_amax_out=amax2, h_out=h2)
    torch.cuda.synchronize()
    return c.cpu().numpy(), h2.cpu().numpy(), q_h, float(g_h), float(amax2.item()), h.cpu().numpy()


# GELU_tanh(c) = c / (1 + 2^X(c)) with X(c) = c (A c^2 + B), B = -2 sqrt(2/pi) log2(e),
# A = 0.044715 B (float64 here; the epilogue evaluates the same form in binary32).
_GELU_B = -2.0 * np.sqrt(2.0 / np.pi) / np.log(2.0)
_GELU_A = 0.044715 * _GELU_B


def gelu_gate_ratios(c, h):
    """Error of the epilogue's FP32 GELU against the float64 formula, as fractions of
    the two gates the design's error analysis gives (both must stay <= 1):
      gate 1: 2^-20 (|c| + |G|)   -- the analysis bounds the error by 2^-22.2 of it;
      gate 2: 2^-20 |G| (1 + w |X|) + 2^-120, w = 2^X / (1 + 2^X): the relative error of
              h, which grows with |X| where h is a small tail value (x = X(c) is formed
              with three binary32 roundings, and h depends on 2^x; about 4 ln2 2^-24 |X|
              w plus ~2^-21.4 from exp2, 1 + e, the reciprocal and the final product),
              and an absolute floor below which the flush-to-zero reciprocal returns 0."""
    c64 = c.astype(np.float64)
    G = oracle.gelu_tanh(c)
    X = c64 * (_GELU_A * c64 * c64 + _GELU_B)
    w = 1.0 / (1.0 + np.exp2(np.minimum(-X, 1000.0)))
    err = np.abs(h.astype(np.float64) - G)
    g1 = 2.0 ** -20 * (np.abs(c64) + np.abs(G))
    g2 = 2.0 ** -20 * np.abs(G) * (1.0 + w * np.abs(X)) + 2.0 ** -120
    with np.errstate(divide="ignore", invalid="ignore"):
        r1 = np.where(err == 0, 0.0, err / g1)
        r2 = np.where(err == 0, 0.0, err / g2)
    return r1, r2


def test_fused_gelu_requant_epilogue(cuda_dev):
    M, N, K = 300, 512, 384
    c, h, q_h, g_h, amax_h, h_cal = fused_case(M, N, K, 24)
    # (i) h is GELU(c) within both gates of the FP32 evaluation's error analysis
    r1, r2 = gelu_gate_ratios(c, h)
    assert r1.max() <= 1.0 and r2.max() <= 1.0, (r1.max(), r2.max())
    assert np.array_equal(h, h_cal)  # deterministic
    # (ii) codes and scales are the oracle's quantization of the GPU's own h with the supplied g
    ref_q = oracle.quantize(h, gscale=g_h)
    codes, scales, g = canonical(q_h)
    assert g == g_h
    assert np.array_equal(scales, ref_q.scales)
    assert np.array_equal(codes, ref_q.codes)
    raw = q_h.scales.cpu().numpy()
    nb = N // 16
    used = np.zeros(raw.size, bool)
    used[[oracle.sf_mma_offset(r, j, N) for r in range(M) for j in range(nb)]] = True
    assert np.all(raw[~used] == 0)
    # (iii) the reported amax is max|h|
    assert amax_h == float(np.abs(h).max())


@pytest.mark.parametrize("M,N", [(512, 512), (128, 256)])  # CTA-pair kernel, single-CTA kernel
def test_gelu_epilogue_tail_and_wide_range(cuda_dev, M, N):
    """c spread over about [-14, 14] (A's tensor scale raised): the negative tail, where
    GELU is a tiny value of c / 2^X, and the positive side where h -> c, both within
    the two gates; h and C from the same call agree with the plain GEMM's c."""
    K = 512
    qx, _ = gpu_quantize(synth.activations(41, M, K), nv.SF_MMA)
    qw, _ = gpu_quantize(synth.weights(41, 0, N, K), nv.SF_MMA)
    c = torch.empty((M, N), dtype=torch.float32, device="cuda")
    nv.nvfp4_gemm(qx, qw, c)
    qx.gscale.mul_(float(np.float32(14.0 / float(c.abs().max()))))
    nv.nvfp4_gemm(qx, qw, c)
    h = torch.empty((M, N), dtype=torch.float32, device="cuda")
    nv.nvfp4_gemm(qx, qw, None, act=nv.ACT_GELU_TANH, h_out=h)
    torch.cuda.synchronize()
    cn, hn = c.cpu().numpy(), h.cpu().numpy()
    assert np.count_nonzero((cn > -10) & (cn < -3)) >= 200
    assert np.count_nonzero(cn > 6) >= 50
    r1, r2 = gelu_gate_ratios(cn, hn)
    print(f"GELU gate ratios M={M} N={N}: gate1 max {r1.max():.3f}, gate2 max {r2.max():.3f}")
    assert r1.max() <= 1.0 and r2.max() <= 1.0, (r1.max(), r2.max())
    assert device_status() == nv.OK


@pytest.mark.slow
def test_fused_ffn_chunk_decomposed(cuda_dev):
    """X 8192 x 3072 -> GEMM to 14336 + GELU + NVFP4 requant -> GEMM to 3072 (bf16).
    Checked by parts on sampled rows: requant bit-exact on the GPU's own h, the
    second GEMM within the bound on the GPU's NVFP4 intermediate."""
    M, K, N = 8192, 3072, 14336
    x = synth.activations(4, M, K)
    w1 = synth.weights(4, 0, N, K)
    w2 = synth.weights(4, 1, K, N)
    qx, _ = gpu_quantize(x, nv.SF_MMA)
    q1, _ = gpu_quantize(w1, nv.SF_MMA)
    q2, _ = gpu_quantize(w2, nv.SF_MMA)
    amax = torch.zeros(1, dtype=torch.float32, device="cuda")
    nv.nvfp4_gemm(qx, q1, None, act=nv.ACT_GELU_TANH, q_amax_out=amax,
                  h_out=torch.empty((M, N), dtype=torch.float32, device="cuda"))
    g_h = float(np.float32(amax.item()) / np.float32(2688.0))
    q_h = nv.NVFP4Tensor(M, N, nv.SF_MMA)
    h = torch.empty((M, N), dtype=torch.float32, device="cuda")
    nv.nvfp4_gemm(qx, q1, None, act=nv.ACT_GELU_TANH, q_out=q_h,
                  q_gscale_in=torch.tensor([g_h], device="cuda"), h_out=h)
    y = torch.empty((M, K), dtype=torch.bfloat16, device="cuda")
    nv.nvfp4_gemm(q_h, q2, y)
    torch.cuda.synchronize()
    rows = np.arange(0, M, 211)
    hs = h.cpu().numpy()[rows]
    ref_q = oracle.quantize(hs, gscale=g_h)
    codes, scales, _ = canonical(q_h)
    assert np.array_equal(codes[rows], ref_q.codes)
    assert np.array_equal(scales[rows], ref_q.scales)
    c2, s2, g2 = canonical(q2)
    ref, bound = oracle.gemm_ref(codes, scales, g_h, c2, s2, g2, rows=rows)
    got = y.float().cpu().numpy()[rows].astype(np.float64)
    assert_within_bound(got, ref, bound, extra_rel=2.0 ** -8)


@pytest.mark.slow
def test_fused_ffn_end_to_end_vs_pure_oracle(cuda_dev):
    """End-to-end report of the fused FFN chunk (X 8192 x 3072 -> 14336 with GELU and
    NVFP4 requantization -> 3072, bf16) against a pure-oracle FFN on sampled rows:
    oracle quantize of X, W1 and W2 -> float64 GEMM of the decoded operands -> FP32 c ->
    float64 GELU -> FP32 h -> oracle quantize with the supplied tensor scale -> float64
    GEMM.  GEMM1 is only bound-exact, so the GPU's h cannot match bit for bit: the
    relative Frobenius error of the output and the mismatch rates of the intermediate's
    codes and scales are printed (the numbers the design notes record) and held to a
    loose sanity bound only.  The supplied scale is an input of the fused epilogue; both
    sides get the same value, RN(max|h| / 2688) of the oracle's h on the sampled rows."""
    M, K, N = 8192, 3072, 14336
    x = synth.activations(4, M, K)
    w1 = synth.weights(4, 0, N, K)
    w2 = synth.weights(4, 1, K, N)
    rows = np.arange(0, M, 257)
    # ---- pure oracle
    qx_o, q1_o, q2_o = oracle.quantize(x), oracle.quantize(w1), oracle.quantize(w2)
    c_o, _ = oracle.gemm_ref(qx_o.codes, qx_o.scales, qx_o.g, q1_o.codes, q1_o.scales, q1_o.g, rows=rows)
    h_o = oracle.gelu_tanh(c_o.astype(np.float32)).astype(np.float32)
    g_h = float(np.float32(np.float32(np.abs(h_o).max()) / np.float32(2688.0)))
    qh_o = oracle.quantize(h_o, gscale=g_h)
    y_o, _ = oracle.gemm_ref(qh_o.codes, qh_o.scales, qh_o.g, q2_o.codes, q2_o.scales, q2_o.g)
    # ---- GPU, through the C ABI
    qx, _ = gpu_quantize(x, nv.SF_MMA)
    q1, _ = gpu_quantize(w1, nv.SF_MMA)
    q2, _ = gpu_quantize(w2, nv.SF_MMA)
    q_h = nv.NVFP4Tensor(M, N, nv.SF_MMA)
    nv.nvfp4_gemm(qx, q1, None, act=nv.ACT_GELU_TANH, q_out=q_h,
                  q_gscale_in=torch.tensor([g_h], dtype=torch.float32, device="cuda"))
    y = torch.empty((M, K), dtype=torch.bfloat16, device="cuda")
    nv.nvfp4_gemm(q_h, q2, y)
    torch.cuda.synchronize()
    assert device_status() == nv.OK
    y_g = y.float().cpu().numpy()[rows].astype(np.float64)
    codes, scales, _ = canonical(q_h)
    nib_g = np.stack([codes[rows] & 0xF, codes[rows] >> 4], axis=-1)
    nib_o = np.stack([qh_o.codes & 0xF, qh_o.codes >> 4], axis=-1)
    rel_fro = float(np.linalg.norm(y_g - y_o) / np.linalg.norm(y_o))
    code_mis = float(np.mean(nib_g != nib_o))
    scale_mis = float(np.mean(scales[rows] != qh_o.scales))
    print(f"fused FFN vs pure-oracle FFN on {len(rows)} rows: relative Frobenius error {rel_fro:.3e}, "
          f"code mismatch rate {code_mis:.3e}, scale mismatch rate {scale_mis:.3e}")
    assert rel_fro < 1e-2 and code_mis < 1e-2 and scale_mis < 1e-2
