"""The Python binding refuses malformed tensors before any pointer reaches the library (CPU only).

The kernels trust the layout they are given (bf16, contiguous, the documented shapes, the current
device); these checks turn a mismatch into MobaError(MOBA_ERR_ARG) instead of a wrong-memory
access. Nothing here launches a kernel: every case fails in the binding's own checks.
"""
import pytest
import torch

from block_sparse_long_moba_b200 import moba


@pytest.fixture
def on_host(monkeypatch):
    """Lets CPU tensors stand in for tensors of the current device, so the shape and dtype checks
    after the device check can be reached without a GPU."""
    monkeypatch.setattr(moba, "_current_device", lambda what, t: t.device)


def _qkv(T=256, hq=4, hkv=2, d=64):
    q = torch.zeros((T, hq, d), dtype=torch.bfloat16)
    k = torch.zeros((T, hkv, d), dtype=torch.bfloat16)
    v = torch.zeros((T, hkv, d), dtype=torch.bfloat16)
    cu = torch.tensor([0, T], dtype=torch.int32)
    return q, k, v, cu


def _raises(fn, text):
    with pytest.raises(moba.MobaError) as ei:
        fn()
    assert ei.value.status == -1
    assert text in str(ei.value)


def test_host_tensors_are_refused():
    q, k, v, cu = _qkv()
    _raises(lambda: moba.moba_attn_fwd(q, k, v, cu, [0, 256], 128, 3), "CUDA")
    _raises(lambda: moba.moba_centroids(k, cu, [0, 256], 128), "CUDA")


def test_dtype_and_contiguity():
    q, k, v, cu = _qkv()
    _raises(lambda: moba.moba_attn_fwd(q.float(), k, v, cu, [0, 256], 128, 3), "bfloat16")
    qt = torch.zeros((4, 256, 64), dtype=torch.bfloat16).transpose(0, 1)
    _raises(lambda: moba.moba_attn_fwd(qt, k, v, cu, [0, 256], 128, 3), "contiguous")
    _raises(lambda: moba.moba_attn_fwd(q[..., 0], k, v, cu, [0, 256], 128, 3), "3-D")


def test_shapes_of_inputs_and_outputs(on_host):
    q, k, v, cu = _qkv()
    call = moba.moba_attn_fwd
    _raises(lambda: call(q, k[:128], v, cu, [0, 256], 128, 3), "k must have shape")
    _raises(lambda: call(q, k, v[:, :1], cu, [0, 256], 128, 3), "v must have shape")
    _raises(lambda: call(q, k, v, cu.long(), [0, 256], 128, 3), "cu_seqlens must be torch.int32")
    _raises(lambda: call(q, k, v, cu, [0, 128, 256], 128, 3), "cu_seqlens must have shape")
    o_bad = torch.zeros((256, 4, 32), dtype=torch.bfloat16)
    _raises(lambda: call(q, k, v, cu, [0, 256], 128, 3, o=o_bad), "o must have shape")
    lse_bad = torch.zeros((256, 4), dtype=torch.float32)
    _raises(lambda: call(q, k, v, cu, [0, 256], 128, 3, lse=lse_bad), "lse must have shape")
    idx_bad = torch.zeros((4, 256, 2), dtype=torch.int32)
    _raises(lambda: call(q, k, v, cu, [0, 256], 128, 3, block_idx_out=idx_bad),
            "block_idx_out must have shape")
    _raises(lambda: call(q, k, v, cu, [0, 256], 128, 3, block_idx_in=idx_bad.float()),
            "block_idx_in must be torch.int32")
    ws_bad = torch.zeros(1024, dtype=torch.float32)
    _raises(lambda: call(q, k, v, cu, [0, 256], 128, 3, workspace=ws_bad), "workspace")
    _raises(lambda: moba.moba_attn_fwd_noalloc(q, k, v, cu, [0, 256], 128, 3, o=o_bad),
            "o must have shape")


def test_centroid_and_gate_buffers(on_host):
    q, k, v, cu = _qkv()
    out_bad = torch.zeros((3, 2, 64), dtype=torch.float32)
    _raises(lambda: moba.moba_centroids(k, cu, [0, 256], 128, out=out_bad), "out must have shape")
    c = torch.zeros((2, 2, 64), dtype=torch.float32)
    _raises(lambda: moba.moba_gate_topk(q, c.double(), cu, [0, 256], 128, 3), "torch.float32")
    _raises(lambda: moba.moba_gate_topk(q, c[:1], cu, [0, 256], 128, 3), "centroids must have")
    idx_bad = torch.zeros((4, 256, 3), dtype=torch.int64)
    _raises(lambda: moba.moba_gate_topk(q, c, cu, [0, 256], 128, 3, out=idx_bad), "torch.int32")
