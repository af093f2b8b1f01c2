"""The Python binding refuses caller buffers that do not match what a call
writes (shape, dtype, device, contiguity) before anything reaches the C ABI,
so a mis-sized `out`, `lse` or workspace can never be overrun on the device."""
import pytest
import torch

import exact_tiled_attention_gqa_b200 as attn

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dev():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda")


def _bf(*shape, dev):
    return torch.zeros(shape, dtype=torch.bfloat16, device=dev)


def test_prefill_results_checked(dev):
    q, k = _bf(1, 8, 64, 128, dev=dev), _bf(1, 2, 64, 128, dev=dev)
    with pytest.raises(ValueError, match="out must have shape"):
        attn.prefill(q, k, k, out=_bf(1, 8, 32, 128, dev=dev))
    with pytest.raises(ValueError, match="lse must have shape"):
        attn.prefill(q, k, k, lse=torch.empty(1, 8, 63, device=dev))
    with pytest.raises(TypeError):
        attn.prefill(q, k, k, lse=torch.empty(1, 8, 64, dtype=torch.float16, device=dev))
    with pytest.raises(ValueError, match="contiguous"):
        attn.prefill(q, k, k, out=_bf(1, 8, 128, 64, dev=dev).transpose(2, 3))


def test_decode_results_and_workspace_checked(dev):
    q, kc = _bf(2, 8, 128, dev=dev), _bf(2, 2, 300, 128, dev=dev)
    sl = torch.tensor([300, 5], dtype=torch.int32, device=dev)
    with pytest.raises(ValueError, match="out must have shape"):
        attn.decode(q, kc, kc, sl, out=_bf(2, 4, 128, dev=dev))
    with pytest.raises(ValueError, match="lse must have shape"):
        attn.decode(q, kc, kc, sl, lse=torch.empty(2, 4, device=dev))
    with pytest.raises(ValueError, match="shape mismatch"):
        attn.decode(q, kc, kc, sl[:1].contiguous())
    # a float32 workspace is sized in bytes, not elements
    need = attn.decode_workspace_size(2, 8, 2, 300, 128)
    ws = torch.empty((need + 3) // 4, dtype=torch.float32, device=dev)
    out, _ = attn.decode(q, kc, kc, sl, workspace=ws)
    torch.cuda.synchronize()
    assert out.shape == q.shape


def test_decode_noalloc_checks(dev):
    q, kc = _bf(2, 8, 128, dev=dev), _bf(2, 2, 300, 128, dev=dev)
    sl = torch.tensor([300, 5], dtype=torch.int32, device=dev)
    with pytest.raises(ValueError, match="out must be given"):
        attn.decode_noalloc(q, kc, kc, sl, out=None)
    with pytest.raises(ValueError, match="out must have shape"):
        attn.decode_noalloc(q, kc, kc, sl, out=_bf(2, 8, 64, dev=dev))
    with pytest.raises(ValueError, match="lse must"):
        attn.decode_noalloc(q, kc, kc, sl, out=torch.empty_like(q), lse=torch.empty(2, device=dev))
    with pytest.raises(ValueError, match="lse must have shape"):
        attn.decode_noalloc(q, kc, kc, sl, out=torch.empty_like(q), lse=torch.empty(2, 4, device=dev))
    with pytest.raises(ValueError, match="shape mismatch"):
        attn.decode_noalloc(q, kc, _bf(2, 2, 299, 128, dev=dev), sl, out=torch.empty_like(q))
    with pytest.raises(ValueError, match="shape mismatch"):
        attn.decode_noalloc(q, _bf(3, 2, 300, 128, dev=dev), _bf(3, 2, 300, 128, dev=dev), sl,
                            out=torch.empty_like(q))


def test_squeezed_decode_results(dev):
    """Decode calls that take q as [B,Hq,D] accept out [B,Hq,D] and lse [B,Hq] as given."""
    q, kp = _bf(2, 8, 128, dev=dev), _bf(4, 2, 64, 128, dev=dev)
    table = torch.tensor([[0, 1], [2, 3]], dtype=torch.int32, device=dev)
    sl = torch.tensor([100, 7], dtype=torch.int32, device=dev)
    out, lse = torch.empty_like(q), torch.empty(2, 8, device=dev)
    o, l = attn.decode_paged(q, kp, kp, table, sl, out=out, lse=lse)
    torch.cuda.synchronize()
    assert o.data_ptr() == out.data_ptr() and l.data_ptr() == lse.data_ptr() and o.shape == q.shape
    with pytest.raises(ValueError, match="out must"):
        attn.decode_paged(q, kp, kp, table, sl, out=_bf(2, 8, 1, 64, dev=dev))
    with pytest.raises(ValueError, match="out must have shape"):
        attn.decode_paged(q, kp, kp, table, sl, out=_bf(2, 8, 64, dev=dev))
