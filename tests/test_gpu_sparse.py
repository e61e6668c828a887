"""GPU parity of sparse absorbed-MLA layers (the lightning-indexer reading: index scores
over a bf16 index-key cache, the top K positions, the latent attention over them) through
the C ABI's layers-only step, against the fp64 CPU oracle.

Bars, per layer and step:
  * index scores: |gpu - oracle| <= bound[t] + 1e-4 max|I|, where
    bound[t] = 2^-8 sum_j |w'_j| sum_i |q_I[j][i] k_I[t][i]| — the queries enter the tensor
    cores rounded to bf16 (relative error <= 2^-9 per entry; the ReLU is 1-Lipschitz), and
    the factor 2 covers the fp32 accumulation and the fp32 projections upstream;
  * chosen positions: exactly the K largest of the GPU's own scores, ties to the lower
    position (an integer decided by floating point: checked in the kernel's precision);
    against the oracle's choice they may differ only at positions whose oracle score is
    within twice the bound of the oracle's K-th score;
  * the layer's output: the oracle run with the GPU's chosen positions, max relative error
    2e-2 (contract) and 1e-4 (regression bound), as for the dense MLA layers;
  * the appended index key and latent row: within one bf16 ulp of the row's largest entry.
Each step feeds both sides the oracle's previous output.
"""
import numpy as np
import pytest

import oracle
from persistent_tile_pipelined_b200.synth import workloads as W

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

from persistent_tile_pipelined_b200 import tre  # noqa: E402

TOL = 2e-2
REG_TOL = 1e-4
ORC = oracle.Oracle(64)

SMALL = W.MLA4.replace(name="mla-sparse-small", n_layers=2, hidden=512, n_q_heads=16,
                       q_lora=128, kv_lora=128, rope_dim=64, nope_dim=64, v_dim=64, prefill=300,
                       decode_steps=3, index_heads=64, index_dim=128, index_topk=64, seed=81)


def relerr(g, o):
    g, o = np.asarray(g, np.float64), np.asarray(o, np.float64)
    return float(np.abs(g - o).max() / max(np.abs(o).max(), 1e-30))


def f64(words):
    return (np.asarray(words, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def np_rms(x, g, eps):
    return x / np.sqrt(np.mean(x * x) + eps) * f64(g)


def score_bound(wl, L, icache, pos, x):
    """2^-8 sum_j |w'_j| sum_i |q_I[j][i] k_I[t][i]| for t in [0, pos], from the layer's
    tensors in fp64 (the cache as the oracle holds it after its append)."""
    HI, DI = wl.index_heads, wl.index_dim
    xn = np_rms(x, L[0], wl.norm_eps)
    cq = np_rms(f64(L[1]) @ xn, L[2], wl.norm_eps)
    kw = f64(L[10]) @ xn
    qi = np.abs((f64(L[9]) @ cq).reshape(HI, DI))
    K = np.abs(f64(icache[: pos + 1]))
    w = np.abs(kw[DI:]) / np.sqrt(HI * DI)
    return 2.0 ** -8 * (w @ (qi @ K.T))


def top_k(scores, k):
    order = np.lexsort((np.arange(scores.size), -scores.astype(np.float64)))
    return set(order[: min(k, scores.size)].tolist())


def dev_words(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def run_sparse(wl, steps=1, mode=None, model=None, **cfg_over):
    model = model or W.gen_mla_model(wl)
    dev = tre.upload_mla_model(model)
    eng = tre.Engine(tre.config_from_workload(wl, debug_flags=tre.TRE_DEBUG_HIDDEN, **cfg_over), dev)
    if mode is not None:
        eng.set_launch_mode(mode)
    caches = [c.copy() for c in model["latent_cache"]]
    icaches = [c.copy() for c in model["index_cache"]]
    x = model["x_in"].astype(np.float64)
    x_dev = torch.empty(wl.hidden, dtype=torch.float32, device="cuda")
    out_dev = torch.empty(wl.hidden, dtype=torch.float32, device="cuda")
    K = wl.index_topk
    stats = {"flips": 0, "worst": 0.0}
    for step in range(steps):
        pos = wl.prefill + step
        x_dev.copy_(torch.from_numpy(x.astype(np.float32)))
        eng.layers_step(x_dev, out_dev, pos)
        torch.cuda.synchronize()
        assert eng.status() == (0, 0)
        hid = eng.hidden().cpu().numpy()
        h = x
        for l in range(wl.n_layers):
            L = model["layers"][l]
            g_sc, g_sel = eng.index(l, pos)
            # the oracle's own scores and choice (on copies of its caches)
            ic_probe = icaches[l].copy()
            _, o_sc, o_sel = ORC.mla_layer_step(wl, L, caches[l].copy(), pos, h,
                                                index_cache=ic_probe, want_index=True)
            bound = score_bound(wl, L, ic_probe, pos, h)
            slack = bound + 1e-4 * np.abs(o_sc).max()
            err = np.abs(g_sc.astype(np.float64) - o_sc)
            assert (err <= slack).all(), \
                f"layer {l} pos {pos}: score err {err.max():.3g} > bound at {int(np.argmax(err - slack))}"
            # the choice: the top K of the GPU's own scores, as a set, no repeats
            assert len(set(g_sel.tolist())) == g_sel.size == min(K, pos + 1)
            assert set(g_sel.tolist()) == top_k(g_sc, K), f"layer {l} pos {pos}: not the top K"
            # against the oracle's choice: only near-ties may differ
            diff = set(g_sel.tolist()) ^ set(o_sel.tolist())
            if diff and pos + 1 > K:
                theta = np.sort(o_sc)[::-1][K - 1]
                near = 2 * slack.max()
                assert all(abs(o_sc[t] - theta) <= near for t in diff), \
                    f"layer {l} pos {pos}: choice differs away from the threshold"
                stats["flips"] += len(diff)
            # the layer output with the GPU's choice
            h = ORC.mla_layer_step(wl, L, caches[l], pos, h, index_cache=icaches[l],
                                   sel=np.sort(g_sel).astype(np.int32))
            e = relerr(hid[l], h)
            stats["worst"] = max(stats["worst"], e)
            assert e <= TOL, f"layer {l} hidden rel err {e:.3g} at pos {pos}"
            assert e <= REG_TOL, f"regression bound: layer {l} hidden rel err {e:.3g} at pos {pos}"
        assert np.array_equal(out_dev.cpu().numpy(), hid[-1])
        x = h
    start, end = wl.prefill, wl.prefill + steps
    for l in range(wl.n_layers):
        for gdev, o in ((dev["k_cache"][l], caches[l]), (dev["v_cache"][l], icaches[l])):
            g = dev_words(gdev)
            assert np.array_equal(g[:start], o[:start])
            gv, ov = f64(g[start:end]), f64(o[start:end])
            row_max = np.abs(ov).max(axis=-1, keepdims=True)
            assert not (np.abs(gv - ov) > 2.0 ** -7 * row_max).any()
    eng.close()
    return stats


@pytest.mark.parametrize("over,steps", [
    (dict(), 3),                                                       # K 64 of 301+
    (dict(index_heads=16, index_dim=64, index_topk=100), 2),           # 1 m-tile, 4 k-steps
    (dict(index_heads=32, index_topk=37, prefill=1000, n_layers=1), 2),  # ragged tiles, odd K
    (dict(kv_lora=512, nope_dim=128, v_dim=128, q_lora=512, hidden=1024, n_q_heads=32,
          prefill=700, index_topk=128, n_layers=1), 2),               # C 576, 2 head groups
], ids=["h64-k64", "h16-d64", "h32-k37", "c576"])
def test_sparse_layers(over, steps):
    run_sparse(SMALL.replace(**over), steps=steps)


def test_sparse_plan_before_and_after_k():
    """pos + 1 <= K attends to every position (the dense path inside the sparse plan);
    the next step, one past K, chooses."""
    run_sparse(SMALL.replace(prefill=63, index_topk=64, decode_steps=3), steps=3)


def test_sparse_small_contexts():
    """Fewer cached positions than scoring splits (most splits score nothing), pos 0."""
    run_sparse(SMALL.replace(prefill=0, index_topk=2, decode_steps=3, n_layers=1), steps=3)
    run_sparse(SMALL.replace(prefill=9, index_topk=4, decode_steps=2, n_layers=1), steps=2)


def test_sparse_ties_go_to_the_lower_position():
    """Duplicated index keys give bit-equal scores; all-zero keys give one score for every
    cached position.  The choice must take the lower positions among equals (the threshold
    bin then holds every candidate, and the pick resolves them by position)."""
    wl = SMALL.replace(n_layers=1, prefill=500, index_topk=48, decode_steps=2)
    model = W.gen_mla_model(wl)
    ic = model["index_cache"][0]
    ic[100:400] = ic[7]                       # 300 equal keys (and one more at 7)
    run_sparse(wl, steps=2, model=model)
    model = W.gen_mla_model(wl)
    model["index_cache"][0][: wl.prefill] = 0  # every cached score 0
    run_sparse(wl, steps=2, model=model)


@pytest.mark.parametrize("cfg", [dict(num_sms=5), dict(num_sms=3, ring_stages=2),
                                 dict(kv_splits=1), dict(gemv_kpart_max=512)],
                         ids=["sms5", "sms3-ring2", "split1", "wo-slices"])
def test_sparse_launch_shapes(cfg):
    run_sparse(SMALL, steps=2, **cfg)


def test_sparse_kernel_per_op_form():
    """Projections, index scoring, selection, attention, W_uv and W_o as separate launches."""
    run_sparse(SMALL, steps=2, mode=tre.TRE_LAUNCH_PER_OP)


@pytest.mark.slow
def test_sparse_full_size_128k():
    """The full workload: hidden 7168, 128 heads, q_lora 1536, kv_lora 512, rope 64, 64 index
    heads of 128, 4 layers over 131072 cached positions, the top 2048 chosen; 2 steps."""
    wl = W.MLA4_SPARSE128K.replace(decode_steps=2)
    stats = run_sparse(wl, steps=2)
    # every flip is already checked to be a near-tie; near-ties stay a small share of K
    # (measured: 66 positions over the 8 choices of 2048, all within the bound)
    assert stats["flips"] <= 0.02 * wl.index_topk * wl.n_layers * 2
