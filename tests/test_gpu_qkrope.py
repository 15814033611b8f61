"""msa_qknorm_rope_insert through the C ABI against the float64 oracle
(oracle/qk_rope_insert.py): normed and rotated queries in place, normed and
rotated keys and raw values written to their page and slot, every other cache
row unchanged."""
import numpy as np
import pytest
import torch

import block_sparse_long_13_b200 as msa
from oracle import qk_rope_insert as R

pytestmark = pytest.mark.gpu

REL, ABS = 8e-3, 2e-3   # bf16 output rounding (2^-9 relative) over fp32 arithmetic


def _case(seed, ctx, nq, num_pages, max_blocks):
    g = torch.Generator().manual_seed(seed)
    S = len(ctx)
    q_start = [0]
    for n in nq:
        q_start.append(q_start[-1] + n)
    T = q_start[-1]
    perm = torch.randperm(num_pages, generator=g)
    pt = torch.full((S, max_blocks), -1, dtype=torch.int32)
    used = 0
    for s in range(S):
        first = (ctx[s] - nq[s]) // 128
        last = (ctx[s] - 1) // 128
        for b in range(first, last + 1):
            pt[s, b] = perm[used]
            used += 1
    batch = msa.Batch.make(q_start, ctx, pt, num_pages)
    pos = np.concatenate([np.arange(c - n, c) for c, n in zip(ctx, nq)])
    seq = np.concatenate([np.full(n, s) for s, n in enumerate(nq)])
    mk = lambda *shape: (torch.randn(*shape, generator=g) * 2).to(torch.bfloat16)
    return dict(batch=batch, pt=pt.numpy(), pos=pos, seq=seq, q=mk(T, 64, 128), k=mk(T, 4, 128), v=mk(T, 4, 128),
                wq=(1 + 0.3 * torch.randn(128, generator=g)).to(torch.bfloat16),
                wk=(1 + 0.3 * torch.randn(128, generator=g)).to(torch.bfloat16),
                kc=mk(num_pages, 4, 128, 128), vc=mk(num_pages, 4, 128, 128))


@pytest.mark.parametrize("theta", [10000.0, 5e6])
@pytest.mark.parametrize("which", ["prefill_and_decode", "positions_near_1m"])
def test_qknorm_rope_insert_matches_oracle(cuda_ok, which, theta):
    if which == "prefill_and_decode":
        c = _case(1, ctx=[300, 1000, 129, 5000], nq=[300, 2, 129, 1], num_pages=64, max_blocks=40)
    else:
        c = _case(2, ctx=[1 << 20, (1 << 20) - 77], nq=[3, 130], num_pages=8, max_blocks=8192)
    cfg = msa.Config()
    q = c["q"].cuda()
    kc, vc = c["kc"].cuda(), c["vc"].cuda()
    msa.qknorm_rope_insert(cfg, c["batch"], q, c["k"].cuda(), c["v"].cuda(), c["wq"].cuda(), c["wk"].cuda(), kc, vc,
                           rotary_dim=64, rope_theta=theta, eps=1e-6)
    assert msa.device_status() == msa.MSA_OK
    q_ref, kc_ref, vc_ref = R.qknorm_rope_insert(c["q"], c["k"], c["v"], c["wq"], c["wk"], c["pos"], c["seq"], c["pt"],
                                                 c["kc"], c["vc"], block_size=128, rotary_dim=64, theta=theta, eps=1e-6)
    got = q.double().cpu().numpy()
    assert np.all(np.abs(got - q_ref) <= REL * np.abs(q_ref) + ABS), float(np.abs(got - q_ref).max())
    kgot, vgot = kc.double().cpu().numpy(), vc.double().cpu().numpy()
    written = np.zeros(kgot.shape[:1] + kgot.shape[2:3], dtype=bool)   # [pages][slot]
    for p, s in zip(c["pos"], c["seq"]):
        written[c["pt"][s][p // 128], p % 128] = True
    w = np.broadcast_to(written[:, None, :, None], kgot.shape)
    assert np.all(np.abs(kgot - kc_ref)[w] <= (REL * np.abs(kc_ref) + ABS)[w])
    assert np.array_equal(vgot[w], vc_ref[w])                          # values are copied bit for bit
    assert np.array_equal(kgot[~w], c["kc"].double().numpy()[~w])     # nothing else is touched
    assert np.array_equal(vgot[~w], c["vc"].double().numpy()[~w])
