"""GPU parity of the quantization step and of the S = Q^ K^^T contraction.

K mean within 1 ulp (in practice identical: binary64 sums of bf16/fp16 inputs are exact),
then codes and scale bytes bit-exact against the oracle fed the GPU's mean; the S tile
against a binary64 product of the oracle-dequantized operands.
"""
import numpy as np
import pytest
import torch

from gpu_helpers import canonical, f32, heads_view
from microscaling_fp4_quantized_b200 import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sage():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import microscaling_fp4_quantized_b200 as s
    s.lib()
    return s


def _compare_quant(sage, oracle_mod, q, k, v, heads=None, smooth_k=True):
    qz = sage.quantize_qkv(q, k, v, smooth_k=smooth_k)
    torch.cuda.synchronize()
    g = canonical(qz)
    assert g["pads_zero"]
    B, H, N, D = q.shape
    hs = list(range(B * H)) if heads is None else list(heads)
    qo, ko, vo = heads_view(q, hs), heads_view(k, hs), heads_view(v, hs)
    if smooth_k:
        km = oracle_mod.kmean(ko)
        ulp = np.abs(g["k_mean"][hs].view(np.int32).astype(np.int64) - km.view(np.int32).astype(np.int64))
        assert ulp.max() <= 1, f"K mean differs by {ulp.max()} ulp"
        o = oracle_mod.quantize_qkv(qo, ko, vo, smooth_k=True, kmean_in=g["k_mean"][hs])
    else:
        o = oracle_mod.quantize_qkv(qo, ko, vo, smooth_k=False)
    for name in ("q_codes", "q_sf", "k_codes", "k_sf", "vt_codes", "vt_sf"):
        got = g[name][hs]
        want = o[name]
        bad = np.argwhere(got != want)
        assert bad.size == 0, f"{name}: {len(bad)} mismatches, first {bad[:5].tolist()} got {got[tuple(bad[0])]} want {want[tuple(bad[0])]}"
    return qz, o


@pytest.mark.parametrize("wl", [
    workloads.TINY,
    workloads.custom(1, 2, 300, 128, seed=11),               # ragged N, bf16
    workloads.custom(2, 1, 77, 64, dtype=torch.float16, seed=12),
    workloads.custom(1, 1, 1, 128, seed=13),                 # one token
    workloads.custom(1, 3, 640, 128, seed=14, outliers=True, bias_sigma=4.0),
], ids=lambda w: w.name)
def test_quant_bit_exact_small(sage, oracle_mod, wl):
    q, k, v = workloads.make_inputs(wl, device="cuda")
    _compare_quant(sage, oracle_mod, q, k, v)


def test_quant_without_smoothing(sage, oracle_mod):
    q, k, v = workloads.make_inputs(workloads.custom(1, 2, 256, 64, seed=15), device="cuda")
    _compare_quant(sage, oracle_mod, q, k, v, smooth_k=False)


@pytest.mark.parametrize("D", [128, 64])
def test_quant_inputs_off_32_byte_boundary(sage, oracle_mod, D):
    """Inputs 16 bytes past a 32-byte boundary (the API asks for 16): the quantizer then
    reads each 16-element block as two 16-byte pieces instead of one 32-byte piece. Codes,
    scales and the K mean must be the same bit for bit."""
    wl = workloads.custom(1, 2, 300, D, seed=16)
    q, k, v = workloads.make_inputs(wl, device="cuda")

    def shifted(t):
        buf = torch.empty(t.numel() + 8, dtype=t.dtype, device=t.device)
        s = buf[8:].view(t.shape)
        s.copy_(t)
        return s

    qs, ks, vs = shifted(q), shifted(k), shifted(v)
    assert qs.data_ptr() % 32 == 16 and ks.data_ptr() % 32 == 16 and vs.data_ptr() % 32 == 16
    _compare_quant(sage, oracle_mod, qs, ks, vs)


def _edge_tensor(D, N, dtype):
    """Blocks built to land on E2M1 and E4M3 rounding ties, signed zeros, saturation,
    subnormal scales and all-zero blocks."""
    rng = np.random.default_rng(5)
    x = np.zeros((N, D), np.float64)
    ties = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 0.0, -0.25, -0.75, -2.5, -5.0, 6.0, -6.0, 0.1, -0.1])
    scales = [1.0, 2.0, 0.5, 2.0 ** -7, 2.0 ** -9, 1.125, 448.0, 3.0]
    for n in range(N):
        for b in range(D // 16):
            kind = (n + b) % 6
            s = scales[(n * 7 + b) % len(scales)]
            if kind == 0:       # element ties under an exact scale (absmax 6 s)
                blk = rng.permutation(ties) * s
            elif kind == 1:     # scale tie: absmax/6 halfway between E4M3 neighbours
                blk = rng.uniform(-1, 1, 16)
                blk[0] = 6.0 * 1.0625 * s
            elif kind == 2:     # saturating scale
                blk = rng.uniform(-3000, 3000, 16)
                blk[3] = 5000.0
            elif kind == 3:     # all zero, with a negative zero
                blk = np.zeros(16)
                blk[1] = -0.0
            elif kind == 4:     # tiny values (scale rounds to 0 or a subnormal)
                blk = rng.uniform(-1, 1, 16) * 6 * 2.0 ** rng.integers(-14, -8)
            else:
                blk = rng.standard_normal(16) * 10.0 ** rng.uniform(-3, 2)
            x[n, 16 * b:16 * b + 16] = blk
    t = torch.from_numpy(x).to(torch.float32).to(dtype)
    return t


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("D", [64, 128])
def test_quant_edge_values(sage, oracle_mod, dtype, D):
    N = 256
    q = _edge_tensor(D, N, dtype)[None, None].contiguous().cuda()
    k = torch.flip(q, dims=[2]).contiguous()
    v = torch.roll(q, 5, dims=2).contiguous()
    _compare_quant(sage, oracle_mod, q, k, v, smooth_k=False)
    _compare_quant(sage, oracle_mod, q, k, v, smooth_k=True)


@pytest.mark.parametrize("wl", [workloads.LONG, workloads.LLM_CAUSAL, workloads.SWEEP[6]],
                         ids=lambda w: w.name)
def test_quant_bit_exact_full_size(sage, oracle_mod, wl):
    # The whole tensor is quantized on the GPU; three heads are checked against the oracle.
    q, k, v = workloads.make_inputs(wl, device="cuda")
    BH = wl.B * wl.H
    _compare_quant(sage, oracle_mod, q, k, v, heads=[0, BH // 2, BH - 1])


@pytest.mark.parametrize("wl", [workloads.TINY, workloads.custom(1, 2, 300, 128, seed=21),
                                workloads.custom(2, 2, 512, 64, seed=22)], ids=lambda w: w.name)
def test_qk_scores_tile(sage, oracle_mod, wl):
    q, k, v = workloads.make_inputs(wl, device="cuda")
    qz = sage.quantize_qkv(q, k, v)
    s = sage.qk_scores(qz, sm_scale=wl.sm_scale)
    torch.cuda.synchronize()
    g = canonical(qz)
    BH, N, D = g["BH"], g["N"], g["D"]

    def deq(codes, sf):
        c = oracle_mod.unpack_fp4(codes)
        return oracle_mod.e2m1_decode(c) * np.repeat(oracle_mod.e4m3_decode(sf), 16, axis=-1)

    qd, kd = deq(g["q_codes"], g["q_sf"]), deq(g["k_codes"], g["k_sf"])
    ref = wl.sm_scale * np.einsum("bnd,bmd->bnm", qd, kd)
    got = s.cpu().numpy()[:, :N, :N].astype(np.float64)
    bound = 1e-5 * wl.sm_scale * np.einsum("bnd,bmd->bnm", np.abs(qd), np.abs(kd)) + 1e-6
    err = np.abs(got - ref)
    assert np.all(err <= bound), f"max err {err.max()} (ref scale {np.abs(ref).max()})"
