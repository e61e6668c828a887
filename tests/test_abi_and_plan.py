"""The C-ABI library loads and exports every declared symbol; the host planner's task
graph is a valid, deadlock-free, balanced partition of the step (no GPU needed)."""
import os
import re
from collections import Counter, defaultdict

import numpy as np
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st
import pytest

from persistent_tile_pipelined_b200 import build
from persistent_tile_pipelined_b200.synth import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

build.build_engine()
from persistent_tile_pipelined_b200 import tre  # noqa: E402

T_GEMV, T_ATTN = 0, 1
OP_QKV, OP_O, OP_GU, OP_DOWN, OP_LM, OP_ROUTER, OP_SGU, OP_RGU, OP_MDOWN = range(9)
OP_MDQKV, OP_UQ, OP_UK, OP_UV, OP_MO, OP_MOS = range(9, 15)
T_MLA_ATTN, T_INDEX, T_ISEL = 2, 3, 4
C_QKV, C_ATTN, C_O, C_GU, C_DOWN, C_ROUTE = range(6)
C_MLA_UK, C_MLA_IDX, C_MLA_SEL = 4, 6, 7
C_PER_LAYER = 8
WHOLE_ROW_OPS = (OP_LM, OP_ROUTER)   # aux holds the op's task count, not K-parts


def declared_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(tre_[a-z_0-9]+)\s*\(", src))
    return names


def test_every_declared_symbol_is_exported():
    names = declared_functions()
    assert {"tre_create", "tre_decode_step", "tre_destroy"} <= names
    for n in names:
        assert hasattr(tre.lib, n), f"{n} declared in include/ but not exported"
    assert set(tre.EXPORTED) == names


def decode_tasks(tasks):
    w0 = tasks[:, 0].astype(np.int64) & 0xFFFFFFFF
    return {
        "type": w0 & 0xFF, "op": (w0 >> 8) & 0xFF, "layer": (w0 >> 16) & 0xFFFF,
        "dep": tasks[:, 1], "dep_count": tasks[:, 2].astype(np.int64) & 0xFFFFFFFF,
        "out": tasks[:, 3], "r0": tasks[:, 4], "r1": tasks[:, 5], "aux": tasks[:, 6],
        "id": tasks[:, 7],
    }


MOE_SMALL = W.MOE4.replace(name="moe-small", n_layers=2, hidden=512, n_q_heads=8, n_kv_heads=2,
                          head_dim=64, prefill=40, n_experts=12, top_k=3, n_shared=1,
                          expert_ffn=200)
MLA_SMALL = W.MLA4.replace(name="mla-small", n_layers=2, hidden=512, n_q_heads=32, q_lora=128,
                          kv_lora=128, rope_dim=64, nope_dim=64, v_dim=64, prefill=100)
MLA_SPARSE = MLA_SMALL.replace(name="mla-sparse-small", prefill=300, index_heads=64, index_dim=128,
                              index_topk=64)
PLAN_CASES = [
    (W.TINY, 148), (W.TINY, 7), (W.LLAMA8B, 148), (W.LLAMA8B, 132),
    (W.TINY.replace(n_q_heads=8, n_kv_heads=1, ffn=696, vocab=1001), 148),
    (W.TINY.replace(n_q_heads=4, n_kv_heads=4, head_dim=128, vocab=77), 33),
    (W.MOE4, 148), (MOE_SMALL, 148), (MOE_SMALL, 5),
    (MOE_SMALL.replace(n_shared=0, top_k=1), 19), (MOE_SMALL.replace(n_shared=2), 64),
    (W.MLA4, 148), (MLA_SMALL, 148), (MLA_SMALL, 6),
    (MLA_SPARSE, 148), (MLA_SPARSE, 6), (W.MLA4_SPARSE128K, 148),
    (MLA_SPARSE.replace(index_heads=16, index_dim=64, index_topk=300), 37),
    # multi-token plans: tensor-core tiles at 4 tokens, CUDA-core rows at 2 and 3
    (W.LLAMA8B.replace(tokens_per_step=4), 148), (W.LLAMA8B.replace(tokens_per_step=2), 148),
    (W.TINY.replace(tokens_per_step=4, hidden=272, ffn=720, vocab=1001), 7),
    (W.TINY.replace(tokens_per_step=3, hidden=264, ffn=696, vocab=1001), 11),
]


def rows_of_ops(wl):
    """Output rows of every GEMV op of one layer."""
    if wl.kind == "mla":
        H = wl.n_q_heads
        rows = {OP_MDQKV: wl.q_lora + wl.kv_lora + wl.rope_dim + wl.index_dim + wl.index_heads,
                OP_UQ: H * (wl.nope_dim + wl.rope_dim) + wl.index_heads * wl.index_dim,
                OP_UK: H * wl.nope_dim,
                OP_UV: H * wl.v_dim, OP_MO: wl.hidden}
        if wl.vocab:
            rows[OP_LM] = wl.vocab
        return rows
    rows = {OP_QKV: (wl.n_q_heads + 2 * wl.n_kv_heads) * wl.head_dim, OP_O: wl.hidden}
    if wl.kind == "moe":
        rows.update({OP_ROUTER: wl.n_experts, OP_RGU: wl.top_k * wl.expert_ffn,
                     OP_MDOWN: wl.hidden})
        if wl.n_shared:
            rows[OP_SGU] = wl.n_shared * wl.expert_ffn
    else:
        rows.update({OP_GU: wl.ffn, OP_DOWN: wl.hidden})
    if wl.vocab:
        rows[OP_LM] = wl.vocab
    return rows


@pytest.mark.parametrize("wl,nsm", PLAN_CASES, ids=lambda x: getattr(x, "name", str(x)))
def test_plan_is_a_valid_task_graph(wl, nsm):
    check_plan(wl, nsm)


def check_plan(wl, nsm, **over):
    """The plan of `wl` on `nsm` SMs is a valid task graph: ids topological per SM queue,
    every dependency produced earlier with the right count, every op's rows covered
    exactly once per K-part, attention (head, split) pairs exactly once, balanced."""
    cfg = tre.config_from_workload(wl, **over)
    tasks, begin = tre.tre_plan_tasks(cfg, num_sms=nsm)
    info = tre.tre_plan_inspect(cfg, num_sms=nsm)
    assert info.num_tasks == len(tasks) and begin[-1] == len(tasks)
    T = decode_tasks(tasks)
    n = len(tasks)
    # ids are a permutation of 0..n-1, increasing within each SM queue (topological order)
    assert sorted(T["id"].tolist()) == list(range(n))
    for s in range(nsm):
        ids = T["id"][begin[s]:begin[s + 1]]
        assert (np.diff(ids) > 0).all()
    # who bumps each counter, and at which global index
    bumpers = defaultdict(list)
    for i in range(n):
        if T["out"][i] >= 0:
            bumpers[int(T["out"][i])].append(i)
    for i in range(n):
        dep = int(T["dep"][i])
        if dep < 0:
            continue
        assert dep < info.num_counters
        producers = bumpers[dep]
        # every producer of a dependency precedes its consumer in global order
        assert all(T["id"][j] < T["id"][i] for j in producers)
        kind = dep % C_PER_LAYER
        if wl.kind == "mla" and kind in (C_MLA_IDX, C_MLA_SEL):
            # sparse: every scoring task bumps the index counter; the selection counter is
            # bumped once, by the selection task that arrives last; attention waits for it
            want = T_INDEX if kind == C_MLA_IDX else T_ISEL
            assert producers and all(T["type"][j] == want for j in producers)
            assert T["dep_count"][i] == (len(producers) if kind == C_MLA_IDX else 1)
            assert T["type"][i] == (T_ISEL if kind == C_MLA_IDX else T_MLA_ATTN)
        elif T["type"][i] == T_GEMV and T["op"][i] == OP_UV:
            # every MLA attention split publishes; W_uv merges a head's splits
            assert T["dep_count"][i] == (wl.n_q_heads // 16) * info.kv_splits
        elif T["type"][i] == T_GEMV and T["op"][i] == OP_O:
            # the attention counter is bumped once per kv head (by the combining split)
            assert T["dep_count"][i] == wl.n_kv_heads
        elif wl.kind == "moe" and kind == C_ROUTE and dep < wl.n_layers * C_PER_LAYER:
            # the route counter is bumped once, by the router task that finishes last
            assert T["dep_count"][i] == 1
            assert producers and all(T["op"][j] == OP_ROUTER for j in producers)
        elif producers and T["op"][producers[0]] == OP_MDOWN:
            # the MoE down counter is bumped once per row block (by its last slot)
            blocks = {int(T["aux"][j]) >> 8 for j in producers}
            assert T["dep_count"][i] == len(blocks)
        elif producers and T["op"][producers[0]] == OP_MOS:
            # the MLA output counter: once per row block (by its last K-slice)
            blocks = {(int(T["aux"][j]) >> 8) & 0xFF for j in producers}
            assert T["dep_count"][i] == len(blocks)
        else:
            assert T["dep_count"][i] == len(producers), (i, dep, kind)
    # every GEMV op's output rows are partitioned exactly once per layer
    rows_of = rows_of_ops(wl)
    whole = np.isin(T["op"], WHOLE_ROW_OPS)
    mdown = T["op"] == OP_MDOWN
    mos = T["op"] == OP_MOS
    part = np.where(whole, 0, T["aux"] & 0xFF)
    nparts = np.where(whole, 1, np.where(mdown, 1, np.where(mos, (T["aux"] >> 16) & 0xFF,
                                                            T["aux"] >> 8)))
    gemv = T["type"] == T_GEMV
    # only the last K-part of a row range publishes (MoE down, MLA output slices: every
    # slot task may; the last to arrive does)
    kp = gemv & ~mdown & ~mos
    assert ((T["out"][kp] >= 0) == (part[kp] == nparts[kp] - 1)).all()
    if wl.kind == "moe":
        # every (slot, row block) pair exactly once; blocks partition the rows
        md = np.flatnonzero(gemv & mdown)
        np_ = wl.n_shared + wl.top_k
        for l in range(wl.n_layers):
            sel = [i for i in md if T["layer"][i] == l]
            pairs = Counter((int(T["aux"][i]) & 0xFF, int(T["aux"][i]) >> 8) for i in sel)
            nb = len({b for _, b in pairs})
            assert set(pairs) == {(j, b) for j in range(np_) for b in range(nb)}
            assert all(v == 1 for v in pairs.values())
            cover = np.zeros(wl.hidden, dtype=np.int64)
            for i in sel:
                if int(T["aux"][i]) & 0xFF == 0:
                    cover[T["r0"][i]:T["r1"][i]] += 1
            assert (cover == 1).all()
        # routed gate/up tasks never straddle two experts; routed work waits for the route
        rg = np.flatnonzero(gemv & (T["op"] == OP_RGU))
        for i in rg:
            assert T["r0"][i] // wl.expert_ffn == (T["r1"][i] - 1) // wl.expert_ffn
            assert T["dep"][i] % C_PER_LAYER == C_ROUTE
        for l in range(wl.n_layers):
            ro = gemv & (T["op"] == OP_ROUTER) & (T["layer"] == l)
            assert (T["aux"][ro] == ro.sum()).all()
    for l in range(wl.n_layers):
        sl = np.flatnonzero(gemv & mos & (T["layer"] == l))
        if len(sl):  # every (slice, block) pair once; blocks partition the rows; 2+ slices
            pairs = Counter((int(T["aux"][i]) & 0xFF, (int(T["aux"][i]) >> 8) & 0xFF) for i in sl)
            ns_ = int(nparts[sl[0]])
            nb = len({b for _, b in pairs})
            assert ns_ >= 2 and set(pairs) == {(j, b) for j in range(ns_) for b in range(nb)}
            cover = np.zeros(wl.hidden, dtype=np.int64)
            for i in sl:
                if int(T["aux"][i]) & 0xFF == 0:
                    cover[T["r0"][i]:T["r1"][i]] += 1
            assert (cover == 1).all()
        for op, N in rows_of.items():
            if op == OP_MDOWN or (op == OP_MO and len(sl)):
                continue
            if op == OP_LM and l != wl.n_layers - 1:
                continue
            sel_op = gemv & (T["op"] == op) & (T["layer"] == l)
            np_op = int(nparts[sel_op][0])
            assert (nparts[sel_op] == np_op).all()
            for pt in range(np_op):
                sel = sel_op & (part == pt)
                cover = np.zeros(N, dtype=np.int64)
                for r0, r1 in zip(T["r0"][sel], T["r1"][sel]):
                    assert 0 <= r0 < r1 <= N
                    cover[r0:r1] += 1
                assert (cover == 1).all(), (l, op, pt)
        sel = (T["type"] == (T_MLA_ATTN if wl.kind == "mla" else T_ATTN)) & (T["layer"] == l)
        pairs = Counter(zip(T["r0"][sel].tolist(), T["r1"][sel].tolist()))
        S = info.kv_splits
        units = wl.n_q_heads // 16 if wl.kind == "mla" else wl.n_kv_heads
        assert set(pairs) == {(g, s) for g in range(units) for s in range(S)}
        assert all(v == 1 for v in pairs.values())
        assert (T["aux"][sel] == S).all()
        for typ in (T_INDEX, T_ISEL):  # sparse: splits 0 .. n - 1 once each, n on every task
            sel = (T["type"] == typ) & (T["layer"] == l)
            if wl.index_topk:
                nsp = int(sel.sum())
                assert nsp >= 1 and sorted(T["r1"][sel].tolist()) == list(range(nsp))
                assert (T["aux"][sel] == nsp).all()
            else:
                assert not sel.any()
    # per layer, attention and MoE-down tasks are spread evenly: no SM holds more than
    # ceil(n / nsm) of one op's tasks (an op ends at a dependency; its slowest SM sets it)
    sm_of = np.zeros(n, dtype=np.int64)
    for q in range(nsm):
        sm_of[T["id"][begin[q]:begin[q + 1]]] = q
    by_id = np.argsort(T["id"])
    for l in range(wl.n_layers):
        for sel in ((T["type"] == T_ATTN), (T["type"] == T_MLA_ATTN), gemv & mdown,
                    gemv & (T["op"] == OP_UK), gemv & (T["op"] == OP_UV)):
            ids = T["id"][sel & (T["layer"] == l)]
            if len(ids):
                counts = np.bincount(sm_of[ids], minlength=nsm)
                assert counts.max() <= -(-len(ids) // nsm), (l, counts.max())
    # tasks that stage residual rows take at most 512 rows (the per-token residual buffer)
    resid_ops = gemv & np.isin(T["op"], (OP_O, OP_DOWN, OP_MO))
    assert ((T["r1"] - T["r0"])[resid_ops] <= 512).all()
    # LM tasks carry the LM task count
    lm = (T["type"] == T_GEMV) & (T["op"] == OP_LM)
    assert (T["aux"][lm] == lm.sum()).all()
    assert info.smem_bytes <= 232448
    return info


@st.composite
def gqa_plans(draw):
    """Random valid GQA stacks and launch shapes (sizes, head groups, SM count, KV
    splits, tokens per step, GEMV form, K-part limit)."""
    D = draw(st.sampled_from([64, 128]))
    kv = draw(st.sampled_from([1, 2, 4, 8]))
    G = draw(st.sampled_from([1, 2, 4, 8]))
    M = draw(st.integers(1, max(1, min(4, 16 // G))))
    form = draw(st.sampled_from([0, 1, 2])) if M > 1 else 0
    q = 16 if form == 2 else 8
    hidden = q * draw(st.integers(4, 256 // (q // 8)))
    ffn = q * draw(st.integers(4, 512 // (q // 8)))
    wl = W.TINY.replace(n_layers=draw(st.integers(1, 3)), hidden=hidden, ffn=ffn,
                        n_kv_heads=kv, n_q_heads=kv * G, head_dim=D,
                        vocab=draw(st.integers(1, 3000)), prefill=draw(st.integers(0, 300)),
                        decode_steps=draw(st.integers(1, 16)), tokens_per_step=M)
    over = {"multi_token_gemv": form}
    kmax = draw(st.sampled_from([0, 512, 1024, 4096]))
    if kmax >= hidden:
        over["gemv_kpart_max"] = kmax
    if draw(st.booleans()):
        over["kv_splits"] = draw(st.integers(1, 4 * D))
    return wl, draw(st.integers(1, 148)), over


@st.composite
def moe_plans(draw):
    """Random valid MoE stacks: expert count, top-k, shared experts, expert width."""
    E = draw(st.integers(1, 64))
    kv = draw(st.sampled_from([1, 2, 4]))
    wl = MOE_SMALL.replace(n_layers=draw(st.integers(1, 2)), hidden=8 * draw(st.integers(8, 96)),
                           n_kv_heads=kv, n_q_heads=kv * draw(st.sampled_from([1, 2, 4, 8])),
                           head_dim=draw(st.sampled_from([64, 128])), n_experts=E,
                           top_k=draw(st.integers(1, min(E, 8))), n_shared=draw(st.integers(0, 2)),
                           expert_ffn=8 * draw(st.integers(1, 64)),
                           prefill=draw(st.integers(0, 200)))
    return wl, draw(st.integers(1, 148)), {}


@st.composite
def moe_fp4_plans(draw):
    """Random valid MoE stacks with MXFP4 routed experts (hidden and expert width multiples
    of 32), on any SM count."""
    wl, nsm, over = draw(moe_plans())
    wl = wl.replace(weight_format="fp4", hidden=32 * draw(st.integers(2, 24)),
                    expert_ffn=32 * draw(st.integers(1, 16)))
    return wl, nsm, over


@st.composite
def mla_plans(draw):
    """Random valid absorbed-MLA stacks: heads, latent and rope widths, q_lora, nope / v."""
    kl = 128 * draw(st.integers(1, 5))
    rope = draw(st.sampled_from([r for r in (16, 32, 48, 64, 80, 96, 112, 128)
                                 if (kl + r) % 64 == 0 and kl + r <= 768] or [64]))
    wl = MLA_SMALL.replace(n_layers=draw(st.integers(1, 2)), hidden=8 * draw(st.integers(8, 96)),
                           n_q_heads=16 * draw(st.integers(1, 4)), kv_lora=kl, rope_dim=rope,
                           q_lora=8 * draw(st.integers(1, 64)), nope_dim=8 * draw(st.integers(1, 16)),
                           v_dim=8 * draw(st.integers(1, 16)), prefill=draw(st.integers(0, 300)))
    return wl, draw(st.integers(1, 148)), {}


@settings(max_examples=60, deadline=None, suppress_health_check=[HealthCheck.too_slow])
@given(st.one_of(moe_plans(), moe_fp4_plans(), mla_plans()))
def test_random_moe_and_mla_plans_are_valid_task_graphs(case):
    wl, nsm, over = case
    check_plan(wl, nsm, **over)


@settings(max_examples=60, deadline=None, suppress_health_check=[HealthCheck.too_slow])
@given(gqa_plans())
def test_random_gqa_plans_are_valid_task_graphs(case):
    wl, nsm, over = case
    info = check_plan(wl, nsm, **over)
    if "kv_splits" in over:
        assert info.kv_splits == over["kv_splits"]


def test_llama8b_plan_is_byte_balanced():
    cfg = tre.config_from_workload(W.LLAMA8B)
    info = tre.tre_plan_inspect(cfg, num_sms=148)
    assert info.kv_splits >= 8
    assert info.ring_stages >= 4
    # every SM streams within 1% of the others over the whole step
    assert info.max_sm_bytes <= 1.01 * info.min_sm_bytes
    assert info.weight_bytes == pytest.approx(15.01e9, rel=0.01)


@pytest.mark.parametrize("field,value,status", [
    ("kind", 1, tre.TRE_ERR_UNSUPPORTED),      # MLA with the GQA config's zero MLA dims
    ("kind", 9, tre.TRE_ERR_INVALID_ARG),
    ("kind", 2, tre.TRE_ERR_UNSUPPORTED),      # MoE with n_experts = 0 (a GQA config)
    ("hidden", 260, tre.TRE_ERR_INVALID_ARG), ("n_kv_heads", 3, tre.TRE_ERR_INVALID_ARG),
    ("head_dim", 96, tre.TRE_ERR_UNSUPPORTED), ("ffn", 690, tre.TRE_ERR_INVALID_ARG),
    ("kv_capacity", 0, tre.TRE_ERR_INVALID_ARG), ("max_tokens_per_step", 5, tre.TRE_ERR_INVALID_ARG),
    ("stage_bytes", 1000, tre.TRE_ERR_INVALID_ARG), ("rope_theta", 0.0, tre.TRE_ERR_INVALID_ARG),
])
def test_plan_rejects_bad_configs(field, value, status):
    cfg = tre.config_from_workload(W.TINY, **{field: value})
    info = tre.tre_plan_info()
    import ctypes
    assert tre.lib.tre_plan_inspect(ctypes.byref(cfg), 148, 232448, ctypes.byref(info)) == status
    assert tre.lib.tre_last_error()


@pytest.mark.parametrize("field,value,status", [
    ("n_experts", 513, tre.TRE_ERR_UNSUPPORTED), ("top_k", 13, tre.TRE_ERR_INVALID_ARG),
    ("top_k", 0, tre.TRE_ERR_INVALID_ARG), ("n_shared", -1, tre.TRE_ERR_INVALID_ARG),
    ("expert_ffn", 100, tre.TRE_ERR_INVALID_ARG),
])
def test_moe_plan_rejects_bad_configs(field, value, status):
    import ctypes
    cfg = tre.config_from_workload(MOE_SMALL, **{field: value})
    info = tre.tre_plan_info()
    assert tre.lib.tre_plan_inspect(ctypes.byref(cfg), 148, 232448, ctypes.byref(info)) == status


def test_moe_plan_streams_only_the_selected_experts():
    wl = W.MOE4
    info = tre.tre_plan_inspect(tre.config_from_workload(wl))
    d, dh = wl.hidden, wl.head_dim
    attn = (wl.n_q_heads + 2 * wl.n_kv_heads) * dh * d + d * wl.n_q_heads * dh
    mlp = wl.n_experts * d + 3 * (wl.n_shared + wl.top_k) * wl.expert_ffn * d
    assert info.weight_bytes == wl.n_layers * ((attn + mlp) * 2 + 2 * d * 2)
    assert info.weight_bytes == pytest.approx(4 * 1.061e9, rel=0.01)
    # levelled up to one MoE-down task (a slot's rows of one row block): 9 slots x 16
    # blocks = 144 tasks on 148 SMs leave 4 SMs without one in the last layer
    nb = 148 // (wl.n_shared + wl.top_k)
    task = -(-wl.hidden // nb) * wl.expert_ffn * 2
    assert info.max_sm_bytes - info.min_sm_bytes <= task + 0.01 * info.min_sm_bytes


@pytest.mark.parametrize("field,value,status", [
    ("n_q_heads", 24, tre.TRE_ERR_UNSUPPORTED), ("kv_lora", 192, tre.TRE_ERR_UNSUPPORTED),
    ("rope_dim", 24, tre.TRE_ERR_UNSUPPORTED), ("rope_dim", 32, tre.TRE_ERR_UNSUPPORTED),
    ("kv_lora", 768, tre.TRE_ERR_UNSUPPORTED), ("v_dim", 12, tre.TRE_ERR_INVALID_ARG),
    ("q_lora", 0, tre.TRE_ERR_INVALID_ARG),
])
def test_mla_plan_rejects_bad_configs(field, value, status):
    import ctypes
    cfg = tre.config_from_workload(MLA_SMALL, **{field: value})
    info = tre.tre_plan_info()
    assert tre.lib.tre_plan_inspect(ctypes.byref(cfg), 148, 232448, ctypes.byref(info)) == status


def test_mla_plan_bytes_and_stage():
    wl = W.MLA4
    info = tre.tre_plan_inspect(tre.config_from_workload(wl))
    H, d, C = wl.n_q_heads, wl.hidden, wl.kv_lora + wl.rope_dim
    w = ((wl.q_lora + C) * d + H * (wl.nope_dim + wl.rope_dim) * wl.q_lora +
         H * wl.nope_dim * wl.kv_lora + H * wl.v_dim * wl.kv_lora + d * H * wl.v_dim)
    assert info.weight_bytes == wl.n_layers * (w * 2 + (d + wl.q_lora + wl.kv_lora) * 2)
    assert info.weight_bytes == pytest.approx(4 * 374.2e6, rel=0.01)
    assert info.stage_bytes == C * 64          # one latent tile of 32 rows per stage
    assert info.ring_stages >= 5
    assert info.kv_bytes_at_capacity == wl.n_layers * wl.prefill * C * 2


@pytest.mark.parametrize("wl,m", [(W.TINY, 2), (W.TINY, 4), (W.LLAMA8B, 4),
                                  (W.TINY.replace(n_q_heads=8, n_kv_heads=1), 2)],
                         ids=["tiny-m2", "tiny-m4", "8b-m4", "g8-m2"])
def test_multi_token_plans(wl, m):
    """M tokens per step: the input planes hold M vectors, so long inputs are cut into
    K-parts of at most 16384 / M floats; the plan still fits one CTA per SM."""
    cfg = tre.config_from_workload(wl, max_tokens_per_step=m)
    info = tre.tre_plan_inspect(cfg)
    tasks, _ = tre.tre_plan_tasks(cfg)
    T = decode_tasks(tasks)
    down = (T["type"] == T_GEMV) & (T["op"] == OP_DOWN)
    kmax = (16384 // m) // 16 * 16
    assert (T["aux"][down] >> 8).max() == -(-wl.ffn // kmax)
    assert info.smem_bytes <= 232448 and info.ring_stages >= 2
    # at 4 tokens the planner picks tensor-core tiles: a stage holds 16 padded row slots
    # of 1024 columns
    if m >= 4:
        assert info.stage_bytes >= 16 * (1024 * 2 + 16)
    resid_ops = (T["type"] == T_GEMV) & np.isin(T["op"], (OP_O, OP_DOWN))
    assert ((T["r1"] - T["r0"])[resid_ops] <= 512).all()
    # the same weights are streamed whatever the token count
    one = tre.tre_plan_inspect(tre.config_from_workload(wl))
    assert info.weight_bytes == one.weight_bytes


@pytest.mark.parametrize("over,status", [
    (dict(max_tokens_per_step=4, n_q_heads=8, n_kv_heads=1), tre.TRE_ERR_UNSUPPORTED),  # 32 rows
    (dict(max_tokens_per_step=2), tre.TRE_ERR_UNSUPPORTED),                            # MoE
    (dict(max_tokens_per_step=4, hidden=264, ffn=696, multi_token_gemv=2),
     tre.TRE_ERR_UNSUPPORTED),                                                          # tiles: K % 16
    (dict(max_tokens_per_step=2, multi_token_gemv=3), tre.TRE_ERR_INVALID_ARG),
])
def test_multi_token_rejections(over, status):
    import ctypes
    base = MOE_SMALL if over == dict(max_tokens_per_step=2) else W.TINY
    cfg = tre.config_from_workload(base, **over)
    info = tre.tre_plan_info()
    assert tre.lib.tre_plan_inspect(ctypes.byref(cfg), 148, 232448, ctypes.byref(info)) == status


def test_multi_token_cuda_core_form_takes_any_k():
    """Whole-row stages (multi_token_gemv = 1, and the planner's choice when the sizes are
    not multiples of 16) need K only a multiple of 8."""
    wl = W.TINY.replace(hidden=264, ffn=696)
    for form in (0, 1):
        info = tre.tre_plan_inspect(tre.config_from_workload(wl, max_tokens_per_step=4,
                                                             multi_token_gemv=form))
        assert info.ring_stages >= 2 and info.stage_bytes < 16 * (1024 * 2 + 16)
    tiled = tre.tre_plan_inspect(tre.config_from_workload(W.TINY, max_tokens_per_step=4))
    rows = tre.tre_plan_inspect(tre.config_from_workload(W.TINY, max_tokens_per_step=4,
                                                         multi_token_gemv=1))
    assert tiled.weight_bytes == rows.weight_bytes
    assert tiled.stage_bytes >= 16 * (1024 * 2 + 16) > rows.stage_bytes
    # two and three tokens: rows by default, tiles on request
    three = tre.tre_plan_inspect(tre.config_from_workload(W.TINY, max_tokens_per_step=3))
    assert three.stage_bytes < 16 * (1024 * 2 + 16)
    two = tre.tre_plan_inspect(tre.config_from_workload(W.TINY, max_tokens_per_step=2))
    two_t = tre.tre_plan_inspect(tre.config_from_workload(W.TINY, max_tokens_per_step=2,
                                                          multi_token_gemv=2))
    assert two.stage_bytes < 16 * (1024 * 2 + 16) <= two_t.stage_bytes


def test_index_fields_are_validated():
    import ctypes
    info = tre.tre_plan_info()

    def status(wl, **over):
        cfg = tre.config_from_workload(wl, **over)
        return tre.lib.tre_plan_inspect(ctypes.byref(cfg), 148, 232448, ctypes.byref(info))

    assert status(MLA_SPARSE) == tre.TRE_OK
    assert status(W.TINY, index_topk=8) == tre.TRE_ERR_INVALID_ARG       # GQA stack
    assert status(MLA_SMALL, index_heads=16) == tre.TRE_ERR_INVALID_ARG  # without a K
    assert status(MLA_SPARSE, index_heads=48) == tre.TRE_ERR_UNSUPPORTED
    assert status(MLA_SPARSE, index_dim=96) == tre.TRE_ERR_UNSUPPORTED
    assert status(MLA_SPARSE, index_topk=MLA_SPARSE.kv_capacity + 1) == tre.TRE_ERR_INVALID_ARG
    assert status(MLA_SPARSE, index_topk=-1) == tre.TRE_ERR_INVALID_ARG


def test_sparse_plan_bytes_follow_the_selection():
    # dense reads every latent row; sparse reads every index key but only K latent rows
    d = tre.tre_plan_inspect(tre.config_from_workload(W.MLA4_KV128K))
    s = tre.tre_plan_inspect(tre.config_from_workload(W.MLA4_SPARSE128K))
    wl = W.MLA4_SPARSE128K
    C, L, cap = wl.kv_lora + wl.rope_dim, wl.n_layers, wl.kv_capacity
    assert d.kv_bytes_at_capacity == L * (cap - 1) * C * 2
    assert s.kv_bytes_at_capacity == L * ((cap - 1) * wl.index_dim * 2 + wl.index_topk * C * 2)
    extra = L * 2 * (wl.index_heads * wl.index_dim * wl.q_lora +
                     (wl.index_dim + wl.index_heads) * wl.hidden)
    assert s.weight_bytes == d.weight_bytes + extra


def test_fault_inject_plans_one_unsatisfiable_wait():
    cfg = tre.config_from_workload(W.TINY, debug_flags=tre.TRE_DEBUG_FAULT_INJECT)
    info = tre.tre_plan_inspect(cfg)
    tasks, _ = tre.tre_plan_tasks(cfg)
    T = decode_tasks(tasks)
    fault_ctr = info.num_counters - 1
    assert (T["dep"] == fault_ctr).sum() == 1
    assert not (T["out"] == fault_ctr).any()


@pytest.mark.parametrize("wl,nsm", PLAN_CASES, ids=lambda x: getattr(x, "name", str(x)))
def test_kernel_per_op_groups(wl, nsm):
    """The kernel-per-op form (TRE_LAUNCH_PER_OP) runs op group g as launch g: every SM's
    queue is covered exactly once, in order, by its ranges of the groups; a group holds the
    tasks of one (layer, type, op); and no task waits on a counter that a task of its own
    or a later group bumps (each launch starts with every dependency of its tasks met, so a
    plain launch cannot deadlock)."""
    cfg = tre.config_from_workload(wl, num_sms=nsm)
    tasks, begin = tre.tre_plan_tasks(cfg, num_sms=148)
    ranges = tre.tre_plan_op_groups(cfg, num_sms=148)
    f = decode_tasks(tasks)
    G = ranges.shape[0]
    assert ranges.shape == (G, nsm, 2)
    group = np.full(len(tasks), -1)
    for s in range(nsm):
        at = begin[s]
        for g in range(G):
            a, b = ranges[g, s]
            if a == b:
                continue
            assert a == at and b > a, "groups must tile the SM queue in order"
            group[a:b] = g
            at = b
        assert at == begin[s + 1]
    assert (group >= 0).all()
    for g in range(G):
        sel = group == g
        key = {(int(t), int(o), int(l)) for t, o, l in zip(f["type"][sel], f["op"][sel], f["layer"][sel])}
        assert len(key) == 1, f"group {g} mixes ops {key}"
    # the last group that bumps each counter (MoE: shared and routed gate/up both bump the
    # gate/up counter; the router's last task bumps the layer's route counter)
    bumped = {}
    for i in range(len(tasks)):
        c = int(f["out"][i])
        if c >= 0:
            bumped[c] = max(bumped.get(c, -1), group[i])
    for i in np.nonzero((f["type"] == T_GEMV) & (f["op"] == OP_ROUTER))[0]:
        c = int(f["layer"][i]) * C_PER_LAYER + C_ROUTE
        bumped[c] = max(bumped.get(c, -1), group[i])
    for i in range(len(tasks)):
        d = int(f["dep"][i])
        if d >= 0:
            assert d in bumped and bumped[d] < group[i], f"task {i} waits inside its launch"
    # launches per step: QKV, attention, O, gate/up, down per GQA layer plus the LM head
    if wl.kind == "gqa":
        assert G == 5 * wl.n_layers + (1 if wl.vocab else 0)


def test_fp8_plans():
    """FP8 projections: the same task graph, every projection row streamed at one byte per
    weight (plus one fp32 scale per 128 x 128 block), the LM head still bf16; the format is
    refused where it is not implemented."""
    fp8 = W.LLAMA8B_FP8
    check_plan(fp8, 148)
    check_plan(W.TINY.replace(weight_format="fp8", hidden=272, ffn=720, vocab=1001), 7)
    info8 = tre.tre_plan_inspect(tre.config_from_workload(fp8))
    info16 = tre.tre_plan_inspect(tre.config_from_workload(W.LLAMA8B))
    d, L, V, F = fp8.hidden, fp8.n_layers, fp8.vocab, fp8.ffn
    nq, nk = fp8.n_q_heads * fp8.head_dim, fp8.n_kv_heads * fp8.head_dim
    proj = (nq + 2 * nk) * d + d * nq + 3 * F * d
    blocks = lambda N, K: -(-N // 128) * -(-K // 128)  # noqa: E731
    scales = 4 * (blocks(nq, d) + 2 * blocks(nk, d) + blocks(d, nq) + 2 * blocks(F, d) + blocks(d, F))
    assert info16.weight_bytes - info8.weight_bytes == L * (proj - scales)
    # byte-balanced over the SMs (within 0.5 % of the busiest SM's bytes)
    assert info8.max_sm_bytes - info8.min_sm_bytes <= 0.005 * info8.max_sm_bytes
    for over, status in [(dict(kind="moe"), tre.TRE_ERR_UNSUPPORTED),
                         (dict(max_tokens_per_step=2), tre.TRE_ERR_UNSUPPORTED),
                         (dict(hidden=264), tre.TRE_ERR_UNSUPPORTED),
                         (dict(weight_format=7), tre.TRE_ERR_INVALID_ARG)]:
        cfg = tre.config_from_workload(W.TINY.replace(weight_format="fp8"))
        for k, v in over.items():
            if k == "kind":
                cfg.kind = tre.TRE_LAYER_MOE
                cfg.n_experts, cfg.top_k, cfg.expert_ffn = 8, 2, 64
            else:
                setattr(cfg, k, v)
        import ctypes
        info = tre.tre_plan_info()
        assert tre.lib.tre_plan_inspect(ctypes.byref(cfg), 148, 232448, ctypes.byref(info)) == status, over


def test_fp4_expert_plans():
    """FP4 routed experts: the same MoE task graph, each selected expert's rows streamed as
    MXFP4 rows (K/2 code bytes + K/32 scale bytes, 16-byte pitch) while attention, router
    and shared expert stay bf16; the format is refused where it is not implemented."""
    from persistent_tile_pipelined_b200.synth import mxfp4_pitch
    fp4 = W.MOE4_FP4
    check_plan(fp4, 148)
    check_plan(MOE_SMALL.replace(weight_format="fp4", hidden=544, expert_ffn=224), 7)
    check_plan(MOE_SMALL.replace(weight_format="fp4", n_shared=0, top_k=1, expert_ffn=96), 19)
    info4 = tre.tre_plan_inspect(tre.config_from_workload(fp4))
    info16 = tre.tre_plan_inspect(tre.config_from_workload(W.MOE4))
    d, Fe, L, k = fp4.hidden, fp4.expert_ffn, fp4.n_layers, fp4.top_k
    assert info16.weight_bytes - info4.weight_bytes == L * k * (
        3 * Fe * d * 2 - 2 * Fe * mxfp4_pitch(d) - d * mxfp4_pitch(Fe))
    # byte-balanced over the SMs (the bf16 shared-expert down slots take the lighter SMs)
    assert info4.max_sm_bytes <= 1.1 * info4.min_sm_bytes
    import ctypes
    for over, status in [(dict(), tre.TRE_OK),
                         (dict(kind=tre.TRE_LAYER_GQA), tre.TRE_ERR_UNSUPPORTED),
                         (dict(max_tokens_per_step=2), tre.TRE_ERR_UNSUPPORTED),
                         (dict(hidden=528), tre.TRE_ERR_UNSUPPORTED),
                         (dict(expert_ffn=200), tre.TRE_ERR_UNSUPPORTED)]:
        cfg = tre.config_from_workload(MOE_SMALL.replace(weight_format="fp4", expert_ffn=224))
        for kk, v in over.items():
            setattr(cfg, kk, v)
        if "kind" in over:
            cfg.ffn = 512
        info = tre.tre_plan_info()
        assert tre.lib.tre_plan_inspect(ctypes.byref(cfg), 148, 232448, ctypes.byref(info)) == status, over
