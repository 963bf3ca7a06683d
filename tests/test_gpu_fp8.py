"""The FP8 gate/up path on the GPU, through the C ABI.

* moe_zc_fp8_quantize_weights (device) equals the host quantiser
  moe_zc_fp8_quantize(MX32) -- itself equal to the FP8 oracle code for code
  -- with the scales laid out in the header's atoms (re-laid out here from
  the row-major host scales by the header's formula).
* moe_zc_forward_fp8 against the fp64 oracle's block-scaled reading
  (oracle/fp8_ref.py, forward_rows_fp8(mx=True): tokens and weights in 1 x 32
  blocks along d with power-of-two scales, gate/up in FP8, down in bf16):
  routing exactly as in the bf16 parity tests, out within the same bounds
  (2e-2 (1 + |ref|) and 5u (|ref| + rms)), and per-expert H and Y rows
  within 2u and 4u of (|ref| + rms): the FP8 products are exact and scaled by
  powers of two, so what is left is fp32 accumulation and the bf16 roundings
  of H, Y and out, as in the bf16 path.
"""
import gc

import numpy as np
import pytest
import torch

from mixture_experts_layer_28_b200 import moe_zc as mz
from mixture_experts_layer_28_b200 import workloads as wl
from oracle import fp8_ref as f8
from oracle import moe_zc_ref as ref
from parity import U, Case, check_output, check_routing

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _free_memory():
    yield
    gc.collect()
    torch.cuda.empty_cache()


# ---------------------------------------------------------------- weights
def _atoms(scales, rows, cols):
    """Host scales (float powers of two, [rows, cols / 32]) as UE8M0 bytes in
    the header's atom order."""
    e = np.log2(scales.astype(np.float64))
    assert np.all(e == np.round(e))
    byte = (np.round(e) + 127).astype(np.int64)
    assert byte.min() >= 0 and byte.max() <= 254
    r = np.arange(rows)[:, None]
    k = np.arange(cols // 32)[None, :]
    off = ((r // 128) * (cols // 128) + k // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + k % 4
    out = np.zeros(rows * cols // 32, dtype=np.uint8)
    out[off.ravel()] = byte.ravel().astype(np.uint8)
    return out


def _weight_cases():
    g = torch.Generator().manual_seed(5)
    yield "gaussian", (torch.randn(256, 384, generator=g) * 0.02).to(torch.bfloat16)
    w = (torch.randn(128, 256, generator=g) * 1e-3).to(torch.bfloat16)
    w[:, :64] = 0.0                                    # all-zero blocks
    w[7, 100] = 1e-30                                  # tiny: subnormal codes
    yield "zeros and tiny", w
    e = torch.randint(-40, 10, (128, 256), generator=g).float()
    yield "wide exponents", (torch.sign(torch.randn(128, 256, generator=g)) * 2.0 ** e).to(torch.bfloat16)
    w = torch.randn(128, 128, generator=g).to(torch.bfloat16)
    w[3, 3] = float("nan")
    w[100, 5] = float("inf")
    yield "non-finite", w
    yield "expert stack", (torch.randn(3, 256, 512, generator=g) * 0.01).to(torch.bfloat16)


@pytest.mark.parametrize("case", [c[0] for c in _weight_cases()])
def test_device_weight_quantiser_matches_host(case):
    W = dict(_weight_cases())[case]
    q = mz.fp8_quantize_weights(W.cuda())
    torch.cuda.synchronize()
    rows, cols = W.numel() // W.shape[-1], W.shape[-1]
    hc, hs = mz.fp8_quantize(W.reshape(rows, cols), mz.FP8_MX32)
    assert np.array_equal(q.codes.reshape(rows, cols).cpu().numpy(), hc), case
    assert np.array_equal(q.scales.cpu().numpy(), _atoms(hs, rows, cols)), case


# ---------------------------------------------------------------- forward
class Fp8Case(Case):
    """A parity case whose gate/up weights are quantised on the device."""

    def __init__(self, w, T=None, bias=None):
        super().__init__(w, T=T, bias=bias)
        self.q_gate = mz.fp8_quantize_weights(self.ew.W_gate)
        self.q_up = mz.fp8_quantize_weights(self.ew.W_up)
        self._oq = {}

    def run_fp8(self):
        d, w = self.dev, self.w
        return mz.forward_fp8(d["x"], d["W_r"], d["b"], self.q_gate, self.q_up, self.ew.W_down,
                              w.N, w.Z, w.K, logit_offset=d["off"])

    def expert_fp8(self, e):
        """The oracle's own quantisation of expert e (block-scaled reading)."""
        if e not in self._oq:
            ew = self.ew
            self._oq[e] = (f8.quantize_mx(ew.W_gate[e].float().cpu().numpy()),
                           f8.quantize_mx(ew.W_up[e].float().cpu().numpy()),
                           ew.W_down[e].double().cpu().numpy())
        return self._oq[e]


def _gpu_fp8(case):
    out = case.run_fp8()
    torch.cuda.synchronize()
    mz.synchronize()
    idx, gate = mz.last_routing(case.T, case.w.K)
    cnt = mz.expert_load(case.w.E)
    return out.float().cpu().numpy().astype(np.float64), idx, gate, cnt


def _check_expert_rows_fp8(case, e, max_rows=64):
    w = case.w
    tok, Hg, Yg, n = mz.last_expert(e, w.d, w.I, max_rows)
    if n == 0:
        return 0
    (gc_, gs), (uc, us), Wd = case.expert_fp8(e)
    xs = case.x[torch.from_numpy(tok.astype(np.int64))].float().numpy()
    cx, sx = f8.quantize_mx(xs)
    Xd = f8.dequantize_blocks(cx, sx, f8.MX_BLOCK)
    a = Xd @ f8.dequantize_blocks(gc_, gs, f8.MX_BLOCK).T
    Ho = ref.silu(a) * (Xd @ f8.dequantize_blocks(uc, us, f8.MX_BLOCK).T)
    Yo = Ho @ Wd.T
    for g, o, name, k in ((Hg.double().numpy(), Ho, "H", 2), (Yg.double().numpy(), Yo, "Y", 4)):
        rms = float(np.sqrt(np.mean(o ** 2)))
        ratio = np.abs(g - o) / (np.abs(o) + rms)
        assert ratio.max() <= k * U, f"expert {e} {name}: max err/(|ref|+rms) {ratio.max():.3e}"
    return n


def _check_fp8(case, rows=None, n_expert_checks=4):
    out_g, idx, gate, cnt = _gpu_fp8(case)
    r_all = case.oracle_routing()
    ok = check_routing(case, r_all, idx, gate, cnt)
    if rows is None:
        rows = np.arange(case.T)
    else:
        rows = rows[ok[rows]]
    sel = torch.from_numpy(rows.astype(np.int64))
    r = case.oracle_routing(rows=sel)
    out_o = f8.forward_rows_fp8(case.x[sel], r, case.expert_fp8, mx=True)
    okr = ok[rows]
    err, rms = check_output(out_g[rows][okr], out_o[okr])
    counts = np.bincount(r_all.idx[r_all.idx < case.w.N].ravel(), minlength=case.w.N)
    order = np.argsort(-counts)
    picks = [int(order[0])] + [int(e) for e in order[::-1] if counts[e] > 0][:n_expert_checks - 1]
    for e in picks:
        _check_expert_rows_fp8(case, e)
    return err, rms


def test_tiny_fp8():
    _check_fp8(Fp8Case(wl.get("tiny")))


def test_small_fp8():
    _check_fp8(Fp8Case(wl.get("small", T=1024)), n_expert_checks=6)


@pytest.mark.parametrize("T", [1, 17, 300])
def test_ragged_token_counts_fp8(T):
    _check_fp8(Fp8Case(wl.get("small", T=T)))


def test_minimum_width_fp8():
    _check_fp8(Fp8Case(wl.get("tiny", d=128, I=128, T=200)))


def test_hot_expert_fp8():
    """One expert with 1100 tokens: FP8 token tiles of 224, 224, 224, 224 and
    204 tokens (two scale atoms each)."""
    w = wl.get("small", T=1100)
    ri = wl.routing_inputs(w, 1100)
    b = ri.b0.clone()
    b[3] += 10.0
    case = Fp8Case(w, T=1100, bias=b)
    _check_fp8(case)
    assert _check_expert_rows_fp8(case, 3, max_rows=1100) == 1100


@pytest.mark.parametrize("over", [dict(d=1024, I=512, T=48), dict(d=384, I=256, T=64, N=40,
                                                                   Z=20, K=6)])
def test_decode_sized_fp8_launch_paths_agree(over):
    """At most 64 tokens: the one grid that also routes, quantises the tokens
    into their slots and combines (the default); the one grid for gate/up
    (FP8) and down (bf16) only; and separate launches: the same bits, and the
    oracle agrees."""
    case = Fp8Case(wl.get("decode", **over))
    res = []
    for path in [dict(off=False, step=True), dict(off=False, step=False), dict(off=True)]:
        mz.test_one_grid(**path)
        try:
            res.append(_gpu_fp8(case))
        finally:
            mz.test_one_grid(False)
    for o, i, _, c in res[1:]:
        assert np.array_equal(res[0][0], o) and np.array_equal(res[0][1], i)
        assert np.array_equal(res[0][3], c)
    _check_fp8(case)


def test_fp8_rejects_widths_off_128():
    """d = 192 is refused (a stage takes 128 contraction elements) before any
    launch; the quantiser refuses such matrices too."""
    w = wl.get("tiny", d=192, I=128, T=16)
    case = Case(w)
    with pytest.raises(mz.MoeZcError) as ei:
        mz.fp8_quantize_weights(case.ew.W_gate)
    assert ei.value.status == mz.ERR_UNSUPPORTED
    codes = torch.zeros(w.N, w.I, w.d, dtype=torch.uint8, device="cuda")
    scales = torch.zeros(w.N * w.I * w.d // 32, dtype=torch.uint8, device="cuda")
    stand_in = mz.Fp8Weight(codes, scales)
    d = case.dev
    with pytest.raises(mz.MoeZcError) as ei:
        mz.forward_fp8(d["x"], d["W_r"], d["b"], stand_in, stand_in, case.ew.W_down,
                       w.N, w.Z, w.K)
    assert ei.value.status == mz.ERR_UNSUPPORTED


@pytest.mark.parametrize("name", ["decode", "prefill"])
def test_full_size_fp8(name):
    case = Fp8Case(wl.get(name))
    rows = wl.tokens_sample(case.T, 128, case.w.seed).numpy()
    _check_fp8(case, rows=rows if case.T > 128 else None, n_expert_checks=3)


def test_logit_offset_fp8():
    """The skewed workload's Zipf logit offset, with FP8 gate/up."""
    _check_fp8(Fp8Case(wl.get("skewed40", T=2048, d=512, I=256)))


def test_fp8_forward_graph_replay():
    """After one eager FP8 forward has sized the workspace, the forward can
    be captured into a CUDA graph; replays equal the eager call bit for bit,
    also after new token values are written into the captured input."""
    case = Fp8Case(wl.get("small", T=512))
    w, d = case.w, case.dev
    out = torch.empty_like(d["x"])
    run = lambda: mz.forward_fp8(d["x"], d["W_r"], d["b"], case.q_gate, case.q_up, case.ew.W_down,
                                 w.N, w.Z, w.K, out=out)
    run()
    torch.cuda.synchronize()
    eager = out.clone()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        run()
    out.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, eager)
    x2 = (torch.randn(w.T, w.d, generator=torch.Generator().manual_seed(9))).to(torch.bfloat16)
    d["x"].copy_(x2.cuda())
    g.replay()
    torch.cuda.synchronize()
    replayed = out.clone()
    run()
    torch.cuda.synchronize()
    assert torch.equal(replayed, out)
    del g


@pytest.mark.parametrize("chunk", [0, 256])
def test_fp8_host_buffer_forward(chunk):
    """moe_zc_forward_host_fp8: with one chunk it equals moe_zc_forward_fp8
    bit for bit; with 256-token chunks each chunk equals moe_zc_forward_fp8
    of that chunk."""
    case = Fp8Case(wl.get("small", T=1000))
    w, d = case.w, case.dev
    x_host = case.x.clone().pin_memory()
    out_host = torch.full_like(x_host, 7.0).pin_memory()
    mz.forward_host_fp8(x_host, d["W_r"], d["b"], case.q_gate, case.q_up, case.ew.W_down,
                        w.N, w.Z, w.K, out_host=out_host, chunk_tokens=chunk or w.T)
    torch.cuda.synchronize()
    mz.synchronize()
    step = chunk or w.T
    for t0 in range(0, w.T, step):
        xs = d["x"][t0:t0 + step].contiguous()
        want = mz.forward_fp8(xs, d["W_r"], d["b"], case.q_gate, case.q_up, case.ew.W_down,
                              w.N, w.Z, w.K)
        torch.cuda.synchronize()
        assert torch.equal(out_host[t0:t0 + step], want.cpu()), t0
