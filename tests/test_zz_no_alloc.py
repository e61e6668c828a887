"""tre_decode_step_static — the decode step for callers that cannot allocate GPU memory.

Some callers cannot call cudaMalloc (code under a framework allocator that must own every
byte, real-time loops that forbid allocation, plug-ins handed only raw pointers).  They
use tre_decode_step_static, which keeps the engine's scratch in a fixed device array
inside the library instead of allocating it.  It runs the same kernel on the same plan as
the regular path (tre_create + tre_decode_step), so the two must agree bit for bit: this
file checks two calls in a row, calls that alternate between two models (the array and
its tensor maps are rewritten in place on every call), that a model too large for the
fixed array is refused before anything runs, and that a call on a capturing stream is
refused.

The file name sorts last so that a run stopping at the first failure has already run
every other test; it also passes alone in a fresh process.
"""
import pytest

from persistent_tile_pipelined_b200.synth import workloads as W

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

from persistent_tile_pipelined_b200 import tre  # noqa: E402


class Pair:
    """One model uploaded twice: a regular engine on one copy, the static path's weights
    table on the other (each path appends to its own KV caches)."""

    def __init__(self, wl):
        self.wl = wl
        model = W.gen_gqa_model(wl)
        self.dev_regular = tre.upload_gqa_model(model)
        self.dev_static = tre.upload_gqa_model(model)
        self.cfg = tre.config_from_workload(wl)
        self.eng = tre.Engine(self.cfg, self.dev_regular)
        self.weights, self.keep = tre.make_weights(self.cfg, self.dev_static)
        self.la = torch.empty(wl.vocab, dtype=torch.float32, device="cuda")
        self.lb = torch.empty(wl.vocab, dtype=torch.float32, device="cuda")
        self.ta = torch.empty(1, dtype=torch.int32, device="cuda")
        self.tb = torch.empty(1, dtype=torch.int32, device="cuda")
        self.tok, self.pos = W.first_token(wl), wl.prefill

    def step_both(self, status):
        stream = torch.cuda.current_stream().cuda_stream
        self.eng.step(self.tok, self.pos, self.la, self.ta)
        st = tre.tre_decode_step_static(self.cfg, self.weights, self.tok, self.pos, stream,
                                        self.lb.data_ptr(), self.tb.data_ptr(),
                                        status.data_ptr())
        assert st == tre.TRE_OK, tre.lib.tre_last_error()
        torch.cuda.synchronize()
        assert status.tolist() == [0, 0]
        assert self.eng.status() == (0, 0)
        # same kernel, plan, launch shape and inputs: identical bits
        assert torch.equal(self.lb, self.la), f"static logits differ at pos {self.pos}"
        assert int(self.tb.item()) == int(self.ta.item())
        self.tok, self.pos = int(self.ta.item()), self.pos + 1

    def check_caches(self):
        for l in range(self.wl.n_layers):
            for name in ("k_cache", "v_cache"):
                a = self.dev_regular[name][l].view(torch.int16)
                b = self.dev_static[name][l].view(torch.int16)
                assert torch.equal(a, b), f"{name}[{l}] differs"

    def close(self):
        self.eng.close()


def test_static_step_matches_regular_step_on_two_calls():
    status = torch.full((2,), 7, dtype=torch.int32, device="cuda")
    pair = Pair(W.TINY)
    for _ in range(2):
        pair.step_both(status)
    pair.check_caches()
    pair.close()


def test_static_step_alternating_two_models():
    """Every call rewrites the plan and the K/V tensor maps at the same addresses in the
    shared array; alternating two models (different weights, caches and shapes) must not
    reuse anything from the previous call."""
    status = torch.full((2,), 7, dtype=torch.int32, device="cuda")
    a = Pair(W.TINY)
    b = Pair(W.TINY.replace(seed=4321, n_kv_heads=4, prefill=100))
    for _ in range(3):
        a.step_both(status)
        b.step_both(status)
    a.check_caches()
    b.check_caches()
    a.close()
    b.close()


def test_static_step_refuses_a_model_beyond_its_fixed_scratch():
    wl = W.TINY.replace(n_layers=300)  # ~7 MB of task descriptors > the 4 MiB array
    cfg = tre.config_from_workload(wl)
    logits = torch.empty(wl.vocab, dtype=torch.float32, device="cuda")
    st = tre.tre_decode_step_static(cfg, tre.tre_weights(), 0, 0, 0, logits.data_ptr(), 0, 0)
    assert st == tre.TRE_ERR_UNSUPPORTED
    assert b"static maximum" in tre.lib.tre_last_error()


def test_static_step_refuses_stream_capture():
    pair = Pair(W.TINY)
    x = torch.zeros(4, device="cuda")
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        with torch.cuda.graph(graph, stream=side):
            x.add_(1.0)
            st = tre.tre_decode_step_static(pair.cfg, pair.weights, pair.tok, pair.pos,
                                            side.cuda_stream, pair.lb.data_ptr(), 0, 0)
    assert st == tre.TRE_ERR_UNSUPPORTED
    assert b"captured" in tre.lib.tre_last_error()
    torch.cuda.synchronize()
    del graph
    pair.close()
