"""GPU checks of the paged AdamW step through the C ABI: each step against the
fp64 oracle evaluated from the GPU's previous state, paged (managed) state
against device-resident state, and a few QLoRA training steps (forward,
backward, AdamW on the flat LoRA parameters) that lower a squared-error loss."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from bit_nf4_quantized_absmax_b200 import binding as b
from bit_nf4_quantized_absmax_b200 import synthetic as syn
from tests.helpers import require_gpu

pytestmark = pytest.mark.gpu

HP = dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8)


def _np(t):
    return t.double().cpu().numpy()


@pytest.mark.parametrize("n", [1, 3, 5, 1027, (1 << 20) + 2])
@pytest.mark.parametrize("wd", [0.0, 0.01])
def test_adamw_step_matches_oracle(n, wd):
    dev = require_gpu()
    gen = torch.Generator().manual_seed(n)
    p = (torch.randn(n, generator=gen) * 0.02).to(dev)
    m = torch.zeros(n, device=dev)
    v = torch.zeros(n, device=dev)
    pb = torch.empty(n, dtype=torch.bfloat16, device=dev)
    for t in range(1, 6):
        g = (torch.randn(n, generator=gen) * 1e-2).to(torch.bfloat16)
        prev = [_np(x) for x in (p, m, v)]
        b.qlora_adamw_step(p, g.to(dev), m, v, t, weight_decay=wd, param_bf16=pb, **HP)
        torch.cuda.synchronize()
        rp, rm, rv = oracle.adamw_step(prev[0], g.float().numpy(), prev[1], prev[2], t, HP["lr"], HP["beta1"],
                                       HP["beta2"], HP["eps"], wd)
        gp, gm, gv = _np(p), _np(m), _np(v)
        # error bounds from the fp32 rounding of each term (a few roundings of 2^-24 each): the
        # first moment can cancel, so its bound scales with its two terms, not with the result
        gf = g.double().numpy()
        b1, b2, lr = (float(np.float32(x)) for x in (HP["beta1"], HP["beta2"], HP["lr"]))
        tol_m = 2.0 ** -21 * (b1 * np.abs(prev[1]) + (1 - b1) * np.abs(gf)) + 1e-30
        tol_v = 2.0 ** -21 * (b2 * prev[2] + (1 - b2) * gf * gf) + 1e-30
        denom = np.sqrt(rv) / np.sqrt(1 - b2 ** t) + float(np.float32(HP["eps"]))
        step = lr / (1 - b1 ** t)
        upd = step * np.abs(rm) / denom
        tol_p = 2.0 ** -21 * (np.abs(prev[0]) + upd) + step * tol_m / denom
        assert np.all(np.abs(gm - rm) <= tol_m), t
        assert np.all(np.abs(gv - rv) <= tol_v), t
        assert np.all(np.abs(gp - rp) <= tol_p), t
        assert torch.equal(pb.cpu(), p.cpu().to(torch.bfloat16))
    assert b.qlora_device_error() == 0


def test_paged_state_gives_the_same_bits_as_device_state():
    dev = require_gpu()
    n = (1 << 21) + 3
    gen = torch.Generator().manual_seed(1)
    p0 = torch.randn(n, generator=gen) * 0.02
    grads = [(torch.randn(n, generator=gen) * 1e-2).to(torch.bfloat16).to(dev) for _ in range(4)]
    # device-resident state
    p_d, m_d, v_d = p0.to(dev), torch.zeros(n, device=dev), torch.zeros(n, device=dev)
    # paged state, moved to host memory between steps (the kernel faults it back)
    bm, bv = b.PagedBuffer(4 * n), b.PagedBuffer(4 * n)
    m_p, v_p = bm.tensor(torch.float32, n), bv.tensor(torch.float32, n)
    m_p.zero_()
    v_p.zero_()
    p_p = p0.to(dev)
    for t, g in enumerate(grads, start=1):
        b.qlora_adamw_step(p_d, g, m_d, v_d, t, weight_decay=0.01, **HP)
        if t % 2:
            bm.prefetch(bm.device)
            bv.prefetch(bv.device)
        b.qlora_adamw_step(p_p, g, m_p, v_p, t, weight_decay=0.01, **HP)
        bm.prefetch(-1)
        bv.prefetch(-1)
    torch.cuda.synchronize()
    assert torch.equal(p_d, p_p) and torch.equal(m_d, m_p) and torch.equal(v_d, v_p)
    assert b.qlora_device_error() == 0
    del m_p, v_p
    bm.free()
    bv.free()


def test_qlora_training_steps_lower_the_loss():
    """Y = X W'^T + s X A^T B^T fitted to a target with only A and B trained."""
    dev = require_gpu()
    N, K, M, r = 256, 512, 64, 16
    inp = syn.make_linear(N, K, M, r=r, alpha=16.0, seed=3, workload="test", dy_std=1.0)
    q = b.qlora_quantize_nf4_dq(inp.W.to(dev))
    X = inp.X.to(dev)
    target = (torch.randn(M, N, generator=torch.Generator().manual_seed(9)) * 0.5).to(torch.bfloat16).to(dev)
    nA, nB = r * K, N * r
    p32 = torch.cat([inp.A.float().reshape(-1), inp.B.float().reshape(-1)]).to(dev)
    pb = p32.to(torch.bfloat16)
    grad = torch.empty(nA + nB, dtype=torch.bfloat16, device=dev)
    m, v = torch.zeros_like(p32), torch.zeros_like(p32)
    A, B = pb[:nA].view(r, K), pb[nA:].view(N, r)
    losses = []
    for t in range(1, 9):
        Y, T = b.qlora_linear_fwd(q, X, A, B, inp.alpha, T_save=True)
        diff = Y.float() - target.float()
        losses.append(0.5 * float((diff * diff).sum()))
        dY = diff.to(torch.bfloat16)
        b.qlora_linear_bwd(q, X, A, B, inp.alpha, dY, T_saved=T, need_dX=False,
                           dA=grad[:nA].view(r, K), dB=grad[nA:].view(N, r))
        b.qlora_adamw_step(p32, grad, m, v, t, lr=1e-2, param_bf16=pb)
    torch.cuda.synchronize()
    assert b.qlora_device_error() == 0
    assert losses[-1] < 0.9 * losses[0], losses
