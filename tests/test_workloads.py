"""The seeded input generators (CPU only): shapes, determinism, and the paged layout's contents."""
import torch

from online_softmax_attention_fwd_b200 import workloads as W


def test_decode_generators_are_deterministic():
    a = W.random_decode(4, 8, 2, 64, [3, 0, 70, 16], seed=7)
    b = W.random_decode(4, 8, 2, 64, [3, 0, 70, 16], seed=7)
    assert torch.equal(a.k, b.k) and torch.equal(a.v, b.v) and torch.equal(a.q, b.q)
    assert a.offsets.tolist() == [0, 3, 3, 73, 89]
    assert a.k.shape == (89, 2, 64) and a.q.shape == (4, 8, 64)


def test_paged_layout_holds_every_key_once_and_nan_elsewhere():
    w = W.random_decode(5, 4, 2, 64, [1, 0, 33, 64, 100], seed=3)
    for page in (16, 32, 64):
        pc = W.paged_from_packed(w, page, seed=page, spare_pages=2)
        num_pages = pc.k_pages.shape[0]
        used = torch.zeros(num_pages, page, dtype=torch.bool)
        off = w.offsets.tolist()
        assert pc.seq_lens.tolist() == [off[n + 1] - off[n] for n in range(5)]
        for n in range(5):
            for t in range(off[n + 1] - off[n]):
                p = int(pc.block_table[n, t // page])
                assert 0 <= p < num_pages and not used[p, t % page]
                used[p, t % page] = True
                assert torch.equal(pc.k_pages[p, t % page], w.k[off[n] + t])
                assert torch.equal(pc.v_pages[p, t % page], w.v[off[n] + t])
        assert int(used.sum()) == off[-1]
        assert torch.isnan(pc.k_pages[~used].float()).all() and torch.isnan(pc.v_pages[~used].float()).all()
        # table entries past a stream's pages are -1 and never needed
        for n in range(5):
            need = (off[n + 1] - off[n] + page - 1) // page
            assert (pc.block_table[n, need:] == -1).all()
