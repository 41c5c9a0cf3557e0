"""Pins of the oracle's attention gradients (routing held fixed), CPU only.

attention_backward is tied to three things other than itself:
  * full limit   -> with topk >= #blocks the layer is causal attention: torch autograd of SDPA in
                    float64 (per sequence; GQA heads expanded, so dK / dV sum over the group);
  * mask form    -> torch autograd in float64 through a dense softmax masked with the routed
                    pattern (the mask-based formulation, MoBA repo radar, "How it works");
  * definition   -> central finite differences of the forward oracle's O with the routing fixed.
A planted mistake (dropping the softmax-row correction D) must fail the mask-form pin.
"""
import math

import numpy as np
import pytest
import torch

from block_sparse_long_moba_b200 import workloads as wl
from oracle import moba_ref as ref


def _inputs(cu, hq, hkv, d, B, topk, keys="offset", seed=0):
    w = wl.custom(cu, hq, hkv, d, B, topk, keys)
    q, k, v, cu_t = wl.make_inputs(w, seed=seed, device="cpu")
    return w, q, k, v


def _d_out(T, H, d, seed=5):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(T, H, d, generator=g, dtype=torch.float64).numpy()


def _masked_autograd(q, k, v, mask, scale, d_out):
    """dQ, dK, dV of sum(dO * O) for O = masked dense softmax attention (torch autograd, fp64)."""
    qt = q.double().clone().requires_grad_(True)
    kt = k.double().clone().requires_grad_(True)
    vt = v.double().clone().requires_grad_(True)
    T, H, d = qt.shape
    r = H // kt.shape[1]
    ke = kt.repeat_interleave(r, dim=1)
    ve = vt.repeat_interleave(r, dim=1)
    z = scale * torch.einsum("thd,uhd->htu", qt, ke)
    z = z.masked_fill(~torch.from_numpy(mask), float("-inf"))
    p = torch.softmax(z, dim=-1)
    o = torch.einsum("htu,uhd->thd", p, ve)
    (o * torch.from_numpy(d_out)).sum().backward()
    return qt.grad.numpy(), kt.grad.numpy(), vt.grad.numpy()


@pytest.mark.parametrize("cu,hq,hkv,d,B", [
    ([0, 64], 1, 1, 16, 16),
    ([0, 50, 50, 121], 4, 2, 8, 16),     # varlen, empty sequence, ragged tails, GQA 2:1
])
def test_backward_full_attention_limit(cu, hq, hkv, d, B):
    w, q, k, v = _inputs(cu, hq, hkv, d, B, 1)
    scale = 1.0 / math.sqrt(d)
    T = cu[-1]
    topk = max(w.seq_blocks()) + 1
    rt, _, _ = ref.forward(q, k, v, cu, B, topk, scale)
    go = _d_out(T, hq, d)
    dq, dk, dv = ref.attention_backward(q, k, v, cu, B, rt.idx, scale, go)
    r = hq // hkv
    for s in range(len(cu) - 1):
        a, b = cu[s], cu[s + 1]
        if a == b:
            continue
        qs = q[a:b].double().permute(1, 0, 2).clone().requires_grad_(True)
        ks = k[a:b].double().permute(1, 0, 2).clone().requires_grad_(True)
        vs = v[a:b].double().permute(1, 0, 2).clone().requires_grad_(True)
        o = torch.nn.functional.scaled_dot_product_attention(
            qs, ks.repeat_interleave(r, dim=0), vs.repeat_interleave(r, dim=0), is_causal=True,
            scale=scale)
        (o * torch.from_numpy(go[a:b]).permute(1, 0, 2)).sum().backward()
        np.testing.assert_allclose(dq[a:b], qs.grad.permute(1, 0, 2).numpy(), atol=1e-11, rtol=1e-9)
        np.testing.assert_allclose(dk[a:b], ks.grad.permute(1, 0, 2).numpy(), atol=1e-11, rtol=1e-9)
        np.testing.assert_allclose(dv[a:b], vs.grad.permute(1, 0, 2).numpy(), atol=1e-11, rtol=1e-9)


@pytest.mark.parametrize("topk", [1, 2, 4])
def test_backward_equals_masked_autograd(topk):
    cu = [0, 61, 61, 150]
    B = 16
    w, q, k, v = _inputs(cu, 4, 2, 16, B, topk, keys="clusters")
    scale = 0.25
    rt, _, _ = ref.forward(q, k, v, cu, B, topk, scale)
    go = _d_out(cu[-1], 4, 16)
    dq, dk, dv = ref.attention_backward(q, k, v, cu, B, rt.idx, scale, go)
    mask = ref.dense_mask(cu, B, rt.idx)
    dq_a, dk_a, dv_a = _masked_autograd(q, k, v, mask, scale, go)
    np.testing.assert_allclose(dq, dq_a, atol=1e-12, rtol=1e-10)
    np.testing.assert_allclose(dk, dk_a, atol=1e-12, rtol=1e-10)
    np.testing.assert_allclose(dv, dv_a, atol=1e-12, rtol=1e-10)


def test_backward_matches_finite_differences():
    cu = [0, 40]
    B = 8
    hq, hkv, d = 2, 1, 4
    w, q, k, v = _inputs(cu, hq, hkv, d, B, 3)
    scale = 0.5
    rt, _, _ = ref.forward(q, k, v, cu, B, 3, scale)
    go = _d_out(cu[-1], hq, d)
    dq, dk, dv = ref.attention_backward(q, k, v, cu, B, rt.idx, scale, go)
    qf, kf, vf = ref.to_f64(q), ref.to_f64(k), ref.to_f64(v)
    toks = np.arange(cu[-1])

    def loss(qx, kx, vx):
        o, _ = ref.attention(qx, kx, vx, cu, B, rt.idx, scale, toks)
        return float((o * go).sum())

    eps = 1e-6
    rng = np.random.default_rng(0)
    for name, arr, grad in (("q", qf, dq), ("k", kf, dk), ("v", vf, dv)):
        for _ in range(6):
            pos = tuple(int(rng.integers(0, n)) for n in arr.shape)
            up, dn = arr.copy(), arr.copy()
            up[pos] += eps
            dn[pos] -= eps
            args_up = {"q": qf, "k": kf, "v": vf}
            args_dn = dict(args_up)
            args_up[name], args_dn[name] = up, dn
            fd = (loss(**{x + "x": args_up[x] for x in "qkv"}) -
                  loss(**{x + "x": args_dn[x] for x in "qkv"})) / (2 * eps)
            assert abs(fd - grad[pos]) <= 1e-6 * max(1.0, abs(fd)), (name, pos, fd, grad[pos])


def test_planted_mistake_in_backward_is_caught(monkeypatch):
    """Dropping the row correction D (dS = p dP instead of p (dP - D)) must fail the mask pin."""
    cu = [0, 48]
    B = 16
    w, q, k, v = _inputs(cu, 2, 1, 8, B, 2)
    rt, _, _ = ref.forward(q, k, v, cu, B, 2, 0.3)
    go = _d_out(cu[-1], 2, 8)
    real_einsum = np.einsum
    monkeypatch.setattr(ref.np, "einsum",
                        lambda spec, *ops, **kw: 0.0 * real_einsum(spec, *ops, **kw)
                        if spec == "thd,thd->ht" else real_einsum(spec, *ops, **kw))
    dq, dk, dv = ref.attention_backward(q, k, v, cu, B, rt.idx, 0.3, go)
    monkeypatch.undo()
    mask = ref.dense_mask(cu, B, rt.idx)
    dq_a, dk_a, dv_a = _masked_autograd(q, k, v, mask, 0.3, go)
    assert not np.allclose(dq, dq_a, atol=1e-6)
    np.testing.assert_allclose(dv, dv_a, atol=1e-12)  # dV does not use D
