"""bench.py's oracle leg times the oracle's own steps only: the selected K / V
blocks are fetched (from the generator or a device cache) between the selection
and the attention, outside the timed region.  The blocks it hands the attention
must give exactly the result of the oracle reading whole sequences."""
import numpy as np
import torch

import bench
from oracle import cpp as C
from workloads import gen


def test_fetched_blocks_give_the_whole_sequence_result():
    C.build()
    wl = gen.make_workload("leg", seed=5, ctx_len=[1500, 700], nq=[1, 2], num_q_heads=16, num_kv_heads=1,
                           idx_heads=4, topk=4, plant_count=1, random_pages=True)
    bs = wl.block_size
    for s in range(wl.num_seqs):
        rows = list(range(wl.q_start[s], wl.q_start[s + 1]))
        pos = wl.positions()[rows].numpy()
        q = gen.query_rows(wl, gen.TID_Q)[rows].float().numpy()
        iq = gen.query_rows(wl, gen.TID_IDX_Q)[rows].float().numpy()
        ctx = torch.arange(wl.ctx_len[s])
        ik = gen.token_tensor(wl, gen.TID_IDX_K, s, ctx).float().numpy()
        kf = gen.token_tensor(wl, gen.TID_K, s, ctx).float().numpy()
        vf = gen.token_tensor(wl, gen.TID_V, s, ctx).float().numpy()
        s64, sel, out, lse = C.msa_rows(q, iq, kf, vf, ik, pos, wl.num_kv_heads, bs, wl.topk, wl.max_blocks)
        k = bench._GenTokens(wl, gen.TID_K, s, "cpu")
        v = bench._GenTokens(wl, gen.TID_V, s, "cpu")
        blocks = sorted(set(int(b) for b in sel[sel >= 0].reshape(-1)))
        assert blocks and blocks[-1] == (wl.ctx_len[s] - 1) // bs      # the last, partial block is among them
        kh = bench._HostBlocks({b: k[b * bs:(b + 1) * bs] for b in blocks}, bs)
        vh = bench._HostBlocks({b: v[b * bs:(b + 1) * bs] for b in blocks}, bs)
        out2, lse2 = C.sparse_attention(q, kh, vh, pos, sel, bs)
        assert np.array_equal(out, out2) and np.array_equal(lse, lse2)
