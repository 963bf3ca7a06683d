"""CUDA path (through the C ABI) against the fp64 oracle on seeded inputs.

Small workloads are compared on every token; the full-size workloads on all
tokens' routing and histogram, and on a seeded sample of output rows that the
oracle computes one by one (rows are independent).  Tolerances: parity.py.
"""
import gc

import numpy as np
import pytest
import torch

from mixture_experts_layer_28_b200 import moe_zc as mz
from mixture_experts_layer_28_b200 import workloads as wl
from oracle import moe_zc_ref as ref
from parity import Case, check_expert_rows, check_output, check_routing

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _free_memory():
    yield
    gc.collect()
    torch.cuda.empty_cache()


def _gpu_result(case):
    out = case.run()
    torch.cuda.synchronize()
    mz.synchronize()
    idx, gate = mz.last_routing(case.T, case.w.K)
    cnt = mz.expert_load(case.w.E)
    return out.float().cpu().numpy().astype(np.float64), idx, gate, cnt


def _full_check(case, n_expert_checks=4):
    out_g, idx, gate, cnt = _gpu_result(case)
    r = case.oracle_routing()
    ok = check_routing(case, r, idx, gate, cnt)
    out_o = ref.forward_rows(case.x, r, case.expert)
    err, rms = check_output(out_g[ok], out_o[ok])
    hit = np.unique(r.idx[r.idx < case.w.N])
    for e in hit[:n_expert_checks]:
        check_expert_rows(case, int(e))
    return err, rms


def _sampled_check(case, n_rows=256, n_expert_checks=3):
    out_g, idx, gate, cnt = _gpu_result(case)
    r_all = case.oracle_routing()
    ok = check_routing(case, r_all, idx, gate, cnt)
    rows = wl.tokens_sample(case.T, n_rows, case.w.seed).numpy()
    rows = rows[ok[rows]]
    r = case.oracle_routing(rows=torch.from_numpy(rows))
    out_o = ref.forward_rows(case.x[torch.from_numpy(rows)], r, case.expert)
    err, rms = check_output(out_g[rows], out_o)
    counts = np.bincount(r_all.idx[r_all.idx < case.w.N].ravel(), minlength=case.w.N)
    # the busiest expert (several GEMM tiles) and a few lightly loaded ones
    order = np.argsort(-counts)
    picks = [int(order[0])] + [int(e) for e in order[::-1] if counts[e] > 0][:n_expert_checks - 1]
    for e in picks:
        check_expert_rows(case, e)
    return err, rms


def test_tiny_full():
    _full_check(Case(wl.get("tiny")))


def test_small_full():
    _full_check(Case(wl.get("small")), n_expert_checks=6)


@pytest.mark.parametrize("T", [1, 17, 300])
def test_ragged_token_counts(T):
    _full_check(Case(wl.get("small", T=T)))


def test_zero_experts_absent():
    """Z = 0: a plain softmax top-K MoE."""
    _full_check(Case(wl.get("small", T=512, Z=0, K=4)))


def test_no_ffn_experts():
    """N = 0: every pick is an identity expert, no GEMM runs; out = (sum g) x."""
    w = wl.get("tiny", N=0, Z=12, K=3)
    case = Case(w)
    out_g, idx, gate, cnt = _gpu_result(case)
    r = case.oracle_routing()
    check_routing(case, r, idx, gate, cnt)
    check_output(out_g, r.zsum[:, None] * case.x.double().numpy())


def test_all_picks_zero_experts_closed_form():
    """Zero experts' bias +10: every pick is a zero expert, out = (sum g) x."""
    w = wl.get("small", T=1000)
    ri = wl.routing_inputs(w, 1000)
    b = ri.b0.clone()
    b[w.N:] += 10.0
    case = Case(w, T=1000, bias=b)
    out_g, idx, gate, cnt = _gpu_result(case)
    assert (idx >= w.N).all()
    assert cnt[: w.N].sum() == 0 and cnt.sum() == 1000 * w.K
    r = case.oracle_routing()
    check_routing(case, r, idx, gate, cnt)
    check_output(out_g, r.zsum[:, None] * case.x.double().numpy())


def test_one_expert_takes_every_token():
    """FFN expert 3 gets all T tokens (several 256-token GEMM tiles)."""
    w = wl.get("small", T=1100)
    ri = wl.routing_inputs(w, 1100)
    b = ri.b0.clone()
    b[3] += 10.0
    case = Case(w, T=1100, bias=b)
    _, _, _, cnt = _gpu_result(case)
    assert cnt[3] == 1100
    _full_check(case)
    assert check_expert_rows(case, 3, max_rows=1100) == 1100


def test_dense_limit_k_equals_e():
    w = wl.get("tiny", T=64, N=6, Z=2, K=8)
    _full_check(Case(w), n_expert_checks=6)


@pytest.mark.parametrize("N,Z,K,over", [
    # E and K both at their largest supported values; with the bias at zero
    # the scores spread the picks over every FFN expert
    (768, 256, 32, dict(bias="zero", w_std=0.05)),
    # every one of the largest expert count is an FFN expert
    (1024, 0, 8, dict(bias="zero", w_std=0.05)),
    (20, 12, 32, {}),   # K = E = 32: dense at the largest K
])
def test_maximum_sizes(N, Z, K, over):
    w = wl.get("tiny", T=300, d=256, I=128, N=N, Z=Z, K=K, **over)
    assert w.E <= mz.MAX_E and w.K <= mz.MAX_K
    _full_check(Case(w), n_expert_checks=6)


def test_minimum_widths():
    w = wl.get("tiny", d=128, I=128, T=200)
    _full_check(Case(w))


def test_odd_weight_blocks():
    """d = 384 and I = 384: the last 256-row weight block is half full."""
    w = wl.get("tiny", d=384, I=384, T=260)
    _full_check(Case(w))


@pytest.mark.parametrize("d", [192, 320])
@pytest.mark.parametrize("T", [260, 48])
def test_widths_not_multiple_of_128(d, T):
    """d % 128 == 64: the down projection's last 128-row weight block is half
    past d (its upper rows are computed but never stored); 48 tokens run the
    two expert GEMMs in one grid, 260 in two launches."""
    _full_check(Case(wl.get("tiny", d=d, I=128, T=T)), n_expert_checks=8)


def test_router_token_tiles_sized_to_waves():
    """40000 tokens fill more than one wave of router tiles, so the router
    GEMM takes 176-token tiles (two full waves instead of 157 tiles of 256):
    ragged last tile and a one-copy box of 176 rows."""
    w = wl.get("tiny", d=128, I=128, T=40000)
    _full_check(Case(w))


def test_paired_tile_launch_matches_plain():
    """Balanced load (experts of ~270 tokens, two token tiles each): once a
    forward has seen such a histogram, the next ones run the expert GEMMs as
    paced 2-CTA clusters.  Every forward gives the same bits, and the oracle
    agrees."""
    w = wl.get("prefill_balanced", T=2048, N=64, Z=32, d=1024, I=256)
    case = Case(w)
    o1, i1, g1, c1 = _gpu_result(case)
    for _ in range(2):
        o2, i2, g2, c2 = _gpu_result(case)
        assert np.array_equal(o1, o2) and np.array_equal(i1, i2) and np.array_equal(c1, c2)
    ffn = c2[: w.N]
    assert 2 * ffn[(ffn > 256) & (ffn <= 512)].sum() >= ffn.sum()   # the balanced shape
    _full_check(case)


@pytest.mark.parametrize("T,d", [(300, 2048), (4096, 2048), (20000, 256)])
def test_exact_ties_pick_lowest_indices(T, d):
    """W_r = 0 and b = 0: every expert scores exactly 1/E, so each token picks
    experts 0..K-1 (ties go to the lower index) with gates 1/E -- through the
    router's K-sliced (few and many tokens) and unsliced route kernels."""
    w = wl.get("small", T=T, d=d, I=128)
    case = Case(w, bias=torch.zeros(w.E))
    case.W_r = torch.zeros_like(case.W_r)
    case.dev["W_r"] = case.W_r.cuda()
    out_g, idx, gate, cnt = _gpu_result(case)
    assert (idx == np.arange(w.K)[None, :]).all()
    assert (gate == np.float32(1.0) / np.float32(w.E)).all()
    want = np.zeros(w.E, dtype=np.int64)
    want[: w.K] = T
    assert np.array_equal(cnt, want)
    r = case.oracle_routing()
    assert (r.idx == np.arange(w.K)[None, :]).all()
    check_output(out_g, ref.forward_rows(case.x, r, case.expert))


def test_empty_batch_is_noop():
    w = wl.get("tiny")
    case = Case(wl.get("tiny", T=1))
    d = case.dev
    x0 = torch.empty(0, w.d, dtype=torch.bfloat16, device="cuda")
    out = torch.full((0, w.d), 1.0, dtype=torch.bfloat16, device="cuda")
    ew = case.ew
    mz.forward(x0, d["W_r"], d["b"], ew.W_gate, ew.W_up, ew.W_down, w.N, w.Z, w.K, out=out)
    torch.cuda.synchronize()
    assert (mz.expert_load(w.E) == 0).all()


def test_deterministic_and_batch_split():
    """Bitwise-equal out, idx, histogram on a rerun; a split batch gives the same rows."""
    w = wl.get("small", T=1024)
    case = Case(w)
    o1, i1, g1, c1 = _gpu_result(case)
    o2, i2, g2, c2 = _gpu_result(case)
    assert np.array_equal(o1, o2) and np.array_equal(i1, i2) and np.array_equal(c1, c2)
    assert np.array_equal(g1, g2)
    d = case.dev
    ew = case.ew
    halves = []
    for sl in (slice(0, 400), slice(400, 1024)):
        halves.append(mz.forward(d["x"][sl].contiguous(), d["W_r"], d["b"], ew.W_gate, ew.W_up,
                                 ew.W_down, w.N, w.Z, w.K).float().cpu().numpy())
    assert np.array_equal(np.concatenate(halves).astype(np.float64), o1)


def test_decode_sized_expert_gemms_match_two_kernel_path():
    """Batches of at most 64 tokens run the gate/up and down tiles in one
    grid (down tiles wait on per-expert counters of finished gate/up tiles);
    their H and Y rows equal, bit for bit, those that the two separate GEMM
    launches of a larger batch compute for the same tokens."""
    w = wl.get("small", T=256)
    case = Case(w)
    d, ew = case.dev, case.ew

    def expert_rows(T):
        mz.forward(d["x"][:T].contiguous(), d["W_r"], d["b"], ew.W_gate, ew.W_up, ew.W_down,
                   w.N, w.Z, w.K)
        torch.cuda.synchronize()
        mz.synchronize()
        rows = {}
        for e in range(w.N):
            tok, H, Y, n = mz.last_expert(e, w.d, w.I, T)
            assert n == len(tok)
            for i, t in enumerate(tok.tolist()):
                rows[(e, t)] = (H[i], Y[i])
        return rows

    fused = expert_rows(64)
    plain = expert_rows(256)
    common = set(fused) & set(plain)
    assert len(fused) > 200 and len(common) >= 0.95 * len(fused)
    for k in common:
        assert torch.equal(fused[k][0], plain[k][0]) and torch.equal(fused[k][1], plain[k][1]), k


# The launch paths of a batch of at most 64 tokens, through the test hook:
# the one grid routing, dispatching, running both expert GEMMs and combining
# (the default: two kernels per forward); the one grid running the expert
# GEMMs only; and separate launches (the path taken when the cooperative
# launch is refused).
PATHS = [dict(off=False, step=True), dict(off=False, step=False), dict(off=True)]


def _result_on_path(case, path, fn):
    mz.test_one_grid(**path)
    try:
        return fn(case)
    finally:
        mz.test_one_grid(False)


@pytest.mark.parametrize("over", [dict(d=1024, I=512), dict(T=1, d=512, I=256),
                                  dict(T=37, d=192, I=256, N=40, Z=20, K=6),
                                  dict(T=64, d=320, I=384, N=24, Z=8, K=8)])
def test_small_batch_launch_paths_give_the_same_bits(over):
    """Output, routing and histogram are the same bits on every path, and
    the default path is the oracle's within the parity bounds."""
    case = Case(wl.get("decode", **over))
    w = case.w
    p = mz.plan(case.T, w.d, w.N, w.Z, w.K, w.I)
    assert p["one_grid_step"] == 1 and p["kernels"] == 2
    res = [_result_on_path(case, path, _gpu_result) for path in PATHS]
    for o, i, g, c in res[1:]:
        assert np.array_equal(res[0][0], o) and np.array_equal(res[0][1], i)
        assert np.array_equal(res[0][2], g) and np.array_equal(res[0][3], c)
    _full_check(case)


def test_small_batch_step_assigns_valid_slots():
    """The slots the one grid assigns: the rows of FFN expert e's range (from
    its first row, count rows) hold exactly the tokens that picked e, each
    once; and those rows' H and Y are the oracle's."""
    case = Case(wl.get("decode", d=512, I=256))
    w = case.w
    _gpu_result(case)
    idx, _ = mz.last_routing(case.T, w.K)
    cnt = mz.expert_load(w.E)[: w.N]
    hit = np.unique(idx[idx < w.N])
    for e in hit:
        tok, _, _, n = mz.last_expert(int(e), w.d, w.I, case.T)
        want = np.nonzero((idx == e).any(axis=1))[0]
        assert n == cnt[e] == len(want)
        assert np.array_equal(np.sort(tok), want)
    for e in hit[:6]:
        check_expert_rows(case, int(e))


def test_one_grid_fallback_gives_the_same_bits():
    """A decode-sized batch with the one grid switched off (the path taken
    when its cooperative launch is refused) gives the same output, routing
    and histogram, bit for bit."""
    case = Case(wl.get("decode", d=1024, I=512))
    assert mz.plan(case.T, case.w.d, case.w.N, case.w.Z, case.w.K,
                   case.w.I)["expert_gemms_one_grid"] == 1
    o1, i1, g1, c1 = _gpu_result(case)
    o2, i2, g2, c2 = _result_on_path(case, dict(off=True), _gpu_result)
    assert np.array_equal(o1, o2) and np.array_equal(i1, i2) and np.array_equal(c1, c2)
    _full_check(case)


def test_logit_offset_moves_routing():
    w = wl.get("skewed40", T=2048, d=512, I=256)
    _full_check(Case(w))


@pytest.mark.parametrize("name", ["decode", "prefill", "decode_balanced", "prefill_balanced"])
def test_full_size_longcat_shaped(name):
    # the balanced companions hit nearly every expert in any sample: fewer rows
    _sampled_check(Case(wl.get(name)), n_rows=128 if name.endswith("balanced") else 256)


@pytest.mark.parametrize("name", ["skewed20", "skewed40", "skewed60"])
def test_full_size_skewed(name):
    _sampled_check(Case(wl.get(name)))


@pytest.mark.parametrize("T,chunk", [(1000, 256), (300, 0), (64, 1000), (2048, 512)])
def test_host_buffer_forward_matches_device_forward(T, chunk):
    """moe_zc_forward_host (chunked copies overlapping compute) gives the same
    bits as moe_zc_forward, and its histogram covers all T tokens."""
    w = wl.get("small", T=T)
    case = Case(w)
    out_d, idx, _, cnt = _gpu_result(case)
    x_host = case.x.clone().pin_memory()
    out_host = torch.full_like(x_host, 7.0).pin_memory()
    ew = case.ew
    d = case.dev
    mz.forward_host(x_host, d["W_r"], d["b"], ew.W_gate, ew.W_up, ew.W_down, w.N, w.Z, w.K,
                    out_host=out_host, chunk_tokens=chunk)
    torch.cuda.synchronize()
    mz.synchronize()
    assert np.array_equal(out_host.float().numpy().astype(np.float64), out_d)
    assert np.array_equal(mz.expert_load(w.E), cnt)


def _bias_hot_expert(w, e, T):
    ri = wl.routing_inputs(w, T)
    b = ri.b0.clone()
    b[e] += 10.0
    return b


@pytest.mark.parametrize("case_id", ["tiny", "ragged17", "hot_expert", "dense", "small"])
def test_expert_gemm_edge_cases(case_id):
    """The expert GEMMs on the edge cases: tiny, 17 tokens (ragged tiles),
    one expert holding 1100 tokens (five token tiles), K = E, and a
    2048-token batch."""
    if case_id == "tiny":
        case = Case(wl.get("tiny"))
    elif case_id == "ragged17":
        case = Case(wl.get("small", T=17))
    elif case_id == "hot_expert":
        w = wl.get("small", T=1100)
        case = Case(w, T=1100, bias=_bias_hot_expert(w, 3, 1100))
    elif case_id == "dense":
        case = Case(wl.get("tiny", T=64, N=6, Z=2, K=8))
    else:
        case = Case(wl.get("small", T=2048))
    _full_check(case, n_expert_checks=6)
    if case_id == "hot_expert":
        assert check_expert_rows(case, 3, max_rows=1100) == 1100


def test_allocation_failure_reports_oom():
    w = wl.get("tiny")
    case = Case(w)
    mz.release()
    mz.test_inject(fail_allocs=1)
    with pytest.raises(mz.MoeZcError) as ei:
        case.run()
    assert ei.value.status == mz.ERR_OOM
    mz.test_inject(0, 0)
    _full_check(case)          # recovers on the next call


@pytest.mark.parametrize("T", [512, 48])
def test_device_wait_timeout_is_reported(T):
    """Bounded device waits given a 1 ns limit give up, report TIMEOUT, and the
    context stays usable for the next forward (48 tokens: the expert GEMMs in
    one grid, whose down tiles also wait on per-expert counters)."""
    w = wl.get("small", T=T)
    case = Case(w)
    case.run()
    mz.synchronize()
    mz.test_inject(0, 1)
    case.run()
    torch.cuda.synchronize()
    with pytest.raises(mz.MoeZcError) as ei:
        mz.synchronize()
    assert ei.value.status == mz.ERR_TIMEOUT
    _full_check(case)
