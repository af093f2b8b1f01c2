"""The device-buffer calls can be captured into a CUDA graph and replayed (the
inner loop of a serving step): after one ordinary call on the device (which sets
each kernel's shared-memory limit), prefill, a prefill that takes the key-split
tail (a merge kernel launched as a programmatic dependent), decode and 8-bit
decode are captured with fixed shapes and buffers, replayed with new inputs copied into those
buffers, and must equal ordinary calls bit for bit."""
import pytest
import torch

import exact_tiled_attention_gqa_b200 as attn
from exact_tiled_attention_gqa_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    attn.device_error(reset=True)
    yield
    assert attn.device_error(reset=True) == 0


def test_capture_and_replay_step():
    dev = torch.device("cuda")
    q, k, v = (t.to(dev) for t in W.prefill_inputs(2, 8, 2, 600, 600, 128, seed=1))
    dq, dk, dv, dsl = W.decode_inputs(4, 32, 8, 3000, 128, 100, 3000, seed=2, device=dev)
    q8, k8, v8, ks8, vs8, sl8 = (t.to(dev) for t in W.decode_inputs_kv8(4, 32, 8, 3000, 128, 100, 3000, W.KV_E4M3,
                                                                         seed=3))
    p_out, p_lse = torch.empty_like(q), torch.empty(2, 8, 600, device=dev)
    d_out, d_lse = torch.empty_like(dq), torch.empty(4, 32, device=dev)
    k_out, k_lse = torch.empty_like(q8), torch.empty(4, 32, 1, device=dev)
    ws = torch.empty(attn.decode_workspace_size(4, 32, 8, 3000, 128), dtype=torch.uint8, device=dev)
    ws8 = torch.empty(attn.decode_kv8_workspace_size(4, 32, 8, 1, 3000, 128), dtype=torch.uint8, device=dev)
    sq, sk, sv = (t.to(dev) for t in W.prefill_inputs(1, 32, 8, 2048, 4096, 128, seed=4))
    s_out, s_lse = torch.empty_like(sq), torch.empty(1, 32, 2048, device=dev)
    pws = torch.empty(attn.prefill_workspace_size(1, 32, 8, 2048, 4096, 128), dtype=torch.uint8, device=dev)
    assert pws.numel() > 0

    def step(stream=None):
        attn.prefill(q, k, v, out=p_out, lse=p_lse, stream=stream)
        attn.prefill(sq, sk, sv, out=s_out, lse=s_lse, workspace=pws, stream=stream)
        attn.decode(dq, dk, dv, dsl, out=d_out, lse=d_lse, workspace=ws, stream=stream)
        attn.decode_kv8(q8, k8, v8, ks8, vs8, sl8, out=k_out, lse=k_lse, workspace=ws8, stream=stream)

    step()                      # first calls: per-kernel setup outside the capture
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        step(stream=s)
    # new inputs in the captured buffers, then replay
    q.copy_(torch.randn_like(q, dtype=torch.float32).to(torch.bfloat16))
    dq.copy_(torch.randn_like(dq, dtype=torch.float32).to(torch.bfloat16))
    q8.copy_(torch.randn_like(q8, dtype=torch.float32).to(torch.bfloat16))
    sq.copy_(torch.randn_like(sq, dtype=torch.float32).to(torch.bfloat16))
    g.replay()
    torch.cuda.synchronize()
    got = [t.clone() for t in (p_out, p_lse, s_out, s_lse, d_out, d_lse, k_out, k_lse)]
    step()
    torch.cuda.synchronize()
    want = (p_out, p_lse, s_out, s_lse, d_out, d_lse, k_out, k_lse)
    assert all(torch.equal(a, b) for a, b in zip(got, want))
    del g


@pytest.mark.parametrize("D", [64, 128])
def test_captured_prefill_and_ordinary_calls_do_not_share_counters(D):
    """A captured prefill keeps one pair of scheduling counters for every replay.
    Ordinary calls cycle through their own 256 pairs, so even with more than 256
    of them running on a second stream while the graph is replayed on a first,
    no launch shares counters with another: every replay gives the captured
    call's exact result, every ordinary call its own, and the device error word
    (which a shared counter would flag) stays clear."""
    dev = torch.device("cuda")
    qa, ka, va = (t.to(dev) for t in W.prefill_inputs(1, 16, 4, 1500, 1500, D, seed=11))
    qb, kb, vb = (t.to(dev) for t in W.prefill_inputs(1, 16, 4, 1100, 1100, D, seed=12))
    want_a, _ = attn.prefill(qa, ka, va)
    want_b, _ = attn.prefill(qb, kb, vb)
    torch.cuda.synchronize()
    out_a = torch.empty_like(qa)
    sa, sb = torch.cuda.Stream(), torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=sa):
        attn.prefill(qa, ka, va, out=out_a, want_lse=False, stream=sa)
    snaps = []
    outs_b = [torch.empty_like(qb) for _ in range(4)]
    n_b = 0
    for i in range(40):
        with torch.cuda.stream(sa):
            g.replay()
            snaps.append(out_a.clone())
        with torch.cuda.stream(sb):
            for _ in range(8):   # 320 ordinary calls in all: every ordinary slot used more than once
                attn.prefill(qb, kb, vb, out=outs_b[n_b % 4], want_lse=False, stream=sb)
                n_b += 1
    torch.cuda.synchronize()
    assert attn.device_error(reset=True) == 0
    assert all(torch.equal(s, want_a) for s in snaps)
    assert all(torch.equal(o, want_b) for o in outs_b)
    del g
