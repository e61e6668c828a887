"""tre_decode_step_static — the decode step for callers that cannot allocate GPU memory.

Some callers cannot call cudaMalloc (code under a framework allocator that must own every
byte, real-time loops that forbid allocation, plug-ins handed only raw pointers).  They
use tre_decode_step_static, which keeps the engine's scratch in a fixed device array
inside the library instead of allocating it.  It must produce the same step as the
regular path (tre_create + tre_decode_step): this file checks two calls in a row on the
same inputs, within the parity tolerance the other GPU tests use, and that a model too
large for the fixed array is refused before anything runs.

The file name sorts last so that a run stopping at the first failure has already run
every other test; it also passes alone in a fresh process.
"""
import numpy as np
import pytest

from persistent_tile_pipelined_b200.synth import workloads as W

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

from persistent_tile_pipelined_b200 import tre  # noqa: E402

TOL = 2e-2  # max |static - regular| / max |regular|, as in the other parity tests


def relerr(g, o):
    g, o = np.asarray(g, np.float64), np.asarray(o, np.float64)
    return float(np.abs(g - o).max() / max(np.abs(o).max(), 1e-30))


def test_static_step_matches_regular_step_on_two_calls():
    wl = W.TINY
    model = W.gen_gqa_model(wl)
    dev_regular = tre.upload_gqa_model(model)  # each path writes its own KV caches
    dev_static = tre.upload_gqa_model(model)
    cfg = tre.config_from_workload(wl)
    eng = tre.Engine(cfg, dev_regular)
    weights, keep = tre.make_weights(cfg, dev_static)
    stream = torch.cuda.current_stream().cuda_stream
    la = torch.empty(wl.vocab, dtype=torch.float32, device="cuda")
    lb = torch.empty(wl.vocab, dtype=torch.float32, device="cuda")
    ta = torch.empty(1, dtype=torch.int32, device="cuda")
    tb = torch.empty(1, dtype=torch.int32, device="cuda")
    status = torch.full((2,), 7, dtype=torch.int32, device="cuda")
    tok, pos = W.first_token(wl), wl.prefill
    for _ in range(2):
        eng.step(tok, pos, la, ta)
        st = tre.tre_decode_step_static(cfg, weights, tok, pos, stream, lb.data_ptr(),
                                        tb.data_ptr(), status.data_ptr())
        assert st == tre.TRE_OK, tre.lib.tre_last_error()
        torch.cuda.synchronize()
        assert status.tolist() == [0, 0]
        assert eng.status() == (0, 0)
        e = relerr(lb.cpu().numpy(), la.cpu().numpy())
        assert e <= TOL, f"static vs regular logits rel err {e:.3g} at pos {pos}"
        assert int(tb.item()) == int(ta.item())
        tok, pos = int(ta.item()), pos + 1
    # the appended KV rows agree too
    for l in range(wl.n_layers):
        for name in ("k_cache", "v_cache"):
            a = dev_regular[name][l][:, wl.prefill:pos].float().cpu().numpy()
            b = dev_static[name][l][:, wl.prefill:pos].float().cpu().numpy()
            assert relerr(b, a) <= TOL
    eng.close()
    del keep


def test_static_step_refuses_a_model_beyond_its_fixed_scratch():
    wl = W.TINY.replace(n_layers=300)  # ~7 MB of task descriptors > the 4 MiB array
    cfg = tre.config_from_workload(wl)
    logits = torch.empty(wl.vocab, dtype=torch.float32, device="cuda")
    st = tre.tre_decode_step_static(cfg, tre.tre_weights(), 0, 0, 0, logits.data_ptr(), 0, 0)
    assert st == tre.TRE_ERR_UNSUPPORTED
    assert b"static maximum" in tre.lib.tre_last_error()
