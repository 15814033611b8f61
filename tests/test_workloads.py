"""The seeded input generator: determinism, layout consistency, statistics."""
import torch

from workloads import configs, gen


def test_hash_is_a_32bit_bijection_sample():
    x = torch.arange(1 << 16, dtype=torch.int64) * 65537
    h = gen.hash32(x & gen.M32)
    assert int(h.min()) >= 0 and int(h.max()) < (1 << 32)
    assert torch.unique(h).numel() == x.numel()


def test_normal_statistics_and_determinism():
    cnt = torch.arange(1 << 20, dtype=torch.int64)
    a = gen.normal_f32(cnt, gen.stream_key(0, gen.TID_K))
    b = gen.normal_f32(cnt, gen.stream_key(0, gen.TID_K))
    c = gen.normal_f32(cnt, gen.stream_key(1, gen.TID_K))
    assert torch.equal(a, b) and not torch.equal(a, c)
    assert abs(float(a.mean())) < 5e-3 and abs(float(a.std()) - 1.0) < 5e-3
    assert float(a.abs().max()) < 3.47  # Irwin-Hall(4) support


def test_paged_cache_matches_logical_order():
    wl = configs.tiny_prefill_2k()
    wl2 = gen.make_workload("t", seed=3, ctx_len=[300, 700], nq=[1, 4], num_q_heads=4,
                            num_kv_heads=2, idx_heads=4, topk=4, plant_count=1, random_pages=True)
    for w in (wl, wl2):
        for tid in (gen.TID_K, gen.TID_V, gen.TID_IDX_K):
            paged = gen.paged_cache(w, tid)
            for s in range(w.num_seqs):
                logical = gen.logical_cache(w, tid, s)
                nb = logical.shape[0] // w.block_size
                pages = w.page_table[s, :nb].long()
                from_pages = paged[pages].permute(0, 2, 1, 3).reshape(logical.shape)
                assert torch.equal(from_pages, logical)


def test_planting_shifts_keys_and_queries():
    wl = configs.tiny_prefill_2k()
    planted = [b for b in range(16) if wl.plant_dir[0][b] >= 0]
    assert len(planted) == 4
    u = wl.dirs(gen.TID_U_IDX, 64)[0].double() * 2  # unit direction
    k = gen.logical_cache(wl, gen.TID_IDX_K, 0).double()
    proj = (k @ u).mean(dim=(1,))  # per token, mean over heads
    blk_mean = proj.view(16, 128).mean(dim=1)
    for b in range(16):
        if b in planted:
            assert blk_mean[b] > 0.35
        else:
            assert abs(float(blk_mean[b])) < 0.15
    q = gen.query_rows(wl, gen.TID_IDX_Q).double()
    assert float((q @ u).mean()) > 0.4


def test_configs_shapes():
    d = configs.decode_128k()
    assert d.total_q == 64 and d.max_blocks == 1024 and d.num_pages == 65536
    assert sorted(d.page_table.flatten().tolist()) == list(range(65536))
    assert all(int((p >= 0).sum()) == 20 for p in d.plant_dir)
    r = configs.verify_ragged()
    assert r.total_q == 128 and all(4096 <= c <= (1 << 20) for c in r.ctx_len)
    ch = configs.chunked_prefill_128k()
    assert [w.ctx_len[0] for w in ch] == [16384 * (c + 1) for c in range(8)]
    assert int((ch[0].plant_dir[0] >= 0).sum()) == 32
    p = configs.prefill_32k()
    assert int((p.plant_dir[0] >= 0).sum()) == 13
