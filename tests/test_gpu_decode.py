"""GPU split-KV decode parity: libattn.so (through its C ABI) vs the fp64 oracle."""
import numpy as np
import pytest
import torch

import online_softmax_attention_fwd_b200 as attn
import oracle
from online_softmax_attention_fwd_b200 import workloads as W
from tests._util import assert_lse, assert_o_bf16, np64, max_abs, running_max_moves

pytestmark = pytest.mark.gpu


def run_decode(w, num_splits=None, max_splits=16, want_lse=True):
    dev = torch.device("cuda")
    q, k, v, off = (t.to(dev) for t in (w.q, w.k, w.v, w.offsets))
    ns = None if num_splits is None else torch.as_tensor(num_splits, dtype=torch.int32, device=dev)
    o, lse = attn.decode(q, k, v, off, num_splits=ns, max_splits=max_splits, scale=w.scale,
                         want_lse=want_lse)
    torch.cuda.synchronize()
    assert attn.device_status() == 0
    return np64(o), (None if lse is None else np64(lse))


def ref(w):
    return oracle.decode_attention(np64(w.q), np64(w.k), np64(w.v), w.offsets.numpy(), w.scale)


def test_decode48():
    w = W.decode48()
    o, lse = run_decode(w)
    assert attn.last_path(2).startswith("decode_splitkv")
    o_ref, lse_ref = ref(w)
    assert_o_bf16(o, o_ref)
    assert_lse(lse, lse_ref)


@pytest.mark.parametrize("lengths,Hq,Hkv,D", [
    ([1, 2, 3, 0, 5, 1000, 257], 8, 2, 128),      # length-1 and empty streams, ragged chunks
    ([4096, 1, 513], 32, 8, 128),
    ([300, 7000, 64], 16, 1, 64),                 # G = 16 (several passes of heads per CTA)
    ([100, 200], 6, 3, 64),                       # G = 2
    ([129, 31], 3, 3, 128),                       # G = 1
    ([2048] * 5, 64, 8, 128),                     # G = 8 at D = 128
])
def test_decode_shapes(lengths, Hq, Hkv, D):
    w = W.random_decode(len(lengths), Hq, Hkv, D, lengths, seed=sum(lengths) + Hq)
    o, lse = run_decode(w)
    o_ref, lse_ref = ref(w)
    assert_o_bf16(o, o_ref)
    assert_lse(lse, lse_ref)


def test_merge_order_only_changes_rounding():
    # the same streams cut into different numbers of chunks give the same result up to rounding
    w = W.random_decode(6, 8, 2, 128, [3000, 1500, 17, 4096, 1024, 2500], seed=11)
    o_ref, lse_ref = ref(w)
    outs = []
    for ns in ([1] * 6, [16] * 6, [3, 7, 1, 13, 2, 9], [64] * 6):
        o, lse = run_decode(w, num_splits=ns, max_splits=64)
        assert_o_bf16(o, o_ref)
        assert_lse(lse, lse_ref)
        outs.append(o)
    for o in outs[1:]:
        assert max_abs(o, outs[0]) <= 2e-2


def test_lse_optional():
    w = W.random_decode(3, 8, 2, 64, [10, 500, 2000], seed=2)
    o, lse = run_decode(w, want_lse=False)
    assert lse is None
    assert_o_bf16(o, ref(w)[0])


def test_empty_stream_gives_zero_and_minus_inf():
    w = W.random_decode(3, 4, 2, 128, [0, 5, 0], seed=4)
    o, lse = run_decode(w)
    assert np.all(o[0] == 0) and np.all(o[2] == 0)
    assert np.all(np.isneginf(lse[0])) and np.all(np.isneginf(lse[2]))


@pytest.mark.parametrize("lengths,Hq,Hkv,D", [
    ([3000, 1500, 700, 4096], 32, 8, 128),
    ([2000, 300, 5000], 8, 8, 64),
])
def test_running_output_rescaled(lengths, Hq, Hkv, D):
    # Keys that grow along each stream make later 16-key blocks of a chunk raise many heads' maximum
    # score by more than 8 (base 2), which is when the split kernel rescales its running (l, o).
    w = W.rising_decode(len(lengths), Hq, Hkv, D, lengths, seed=len(lengths) + D)
    qn, kn, off = np64(w.q), np64(w.k), w.offsets.numpy()
    G = Hq // Hkv
    moved = []
    for n, L in enumerate(lengths):
        C = attn.default_splits(L, 16)
        chunk = -(-L // C)
        for c in range(C):
            s0, s1 = int(off[n]) + c * chunk, int(off[n]) + min(L, (c + 1) * chunk)
            if s1 <= s0:
                continue
            x = np.stack([w.scale * kn[s0:s1, h // G] @ qn[n, h] for h in range(Hq)])
            moved.append(running_max_moves(x, 16) > 0)
    moved = np.concatenate(moved)
    assert moved.mean() > 0.25 and (~moved).mean() > 0.05, moved.mean()
    o, lse = run_decode(w)
    o_ref, lse_ref = ref(w)
    assert_o_bf16(o, o_ref)
    assert_lse(lse, lse_ref)


# ---------------------------------------------------------------------------------------------
# Several query tokens per stream (attn_decode_splitkv_qlen): token t of a stream with L keys sees
# keys 0 .. L - q_len + t.
# ---------------------------------------------------------------------------------------------

def ref_qlen(w):
    return oracle.decode_attention_qlen(np64(w.q), np64(w.k), np64(w.v), w.offsets.numpy(), w.scale)


@pytest.mark.parametrize("lengths,q_len,Hq,Hkv,D", [
    ([1000, 2, 513, 0, 64], 2, 32, 8, 128),     # 4 heads x 2 tokens per item (8 of 16 rows)
    ([700, 3000, 5, 4096], 4, 32, 8, 128),      # 4 heads x 4 tokens (16 rows)
    ([300, 1, 2048], 3, 8, 8, 64),              # one head x 3 tokens (the 4-row variant)
    ([1500, 17, 800], 8, 8, 2, 128),            # two token passes per head group
    ([900, 33], 16, 6, 3, 64),                  # 2 heads x 8 tokens, two passes
    ([4096, 2000], 5, 16, 1, 128),              # G = 16: four head passes, a partial token pass
    ([50, 10, 0], 20, 4, 4, 64),                # more tokens than 16 rows; L < q_len for one stream
])
def test_decode_qlen(lengths, q_len, Hq, Hkv, D):
    w = W.random_decode(len(lengths), Hq, Hkv, D, lengths, seed=sum(lengths) + q_len, q_len=q_len)
    o, lse = run_decode(w)
    assert attn.last_path(2) == "decode_splitkv_qlen_mma16816"
    assert o.shape == (len(lengths), q_len, Hq, D) and lse.shape == (len(lengths), Hq, q_len)
    o_ref, lse_ref = ref_qlen(w)
    assert_o_bf16(o, o_ref)
    assert_lse(lse, lse_ref)


def test_decode_qlen_rising_keys_and_split_counts():
    # rows that rescale their running output, cut into different numbers of chunks
    w = W.rising_decode(4, 32, 8, 128, [3000, 1500, 700, 4096], seed=7, q_len=4)
    o_ref, lse_ref = ref_qlen(w)
    for ns in (None, [1, 3, 16, 64]):
        o, lse = run_decode(w, num_splits=ns, max_splits=64 if ns else 16)
        assert_o_bf16(o, o_ref)
        assert_lse(lse, lse_ref)


def test_decode_qlen_one_token_equals_decode():
    w3 = W.random_decode(5, 32, 8, 128, [100, 2000, 0, 1, 4096], seed=8)
    w4 = W.random_decode(5, 32, 8, 128, [100, 2000, 0, 1, 4096], seed=8, q_len=1)
    o3, l3 = run_decode(w3)
    o4, l4 = run_decode(w4)
    assert np.array_equal(o3, o4[:, 0]) and np.array_equal(l3, l4[..., 0])


def test_decode_qlen_paged():
    w = W.random_decode(5, 32, 8, 128, [1000, 3, 64, 4096, 77], seed=9, q_len=4)
    o, lse, pc = run_paged(w, 64, seed=2)
    assert attn.device_status() == 0
    assert attn.last_path(2) == "decode_splitkv_paged_qlen_mma16816"
    assert np.all(np.isfinite(o))
    o_ref, lse_ref = oracle.decode_attention_paged_qlen(np64(w.q), np64(pc.k_pages), np64(pc.v_pages),
                                                        pc.block_table.numpy(), pc.seq_lens.numpy(), w.scale)
    assert_o_bf16(o, o_ref)
    assert_lse(lse, lse_ref)


# ---------------------------------------------------------------------------------------------
# Paged caches (attn_decode_paged): the same streams read through a block table from a shuffled
# pool whose unused rows are NaN.
# ---------------------------------------------------------------------------------------------

def run_paged(w, page_size, seed=0, num_splits=None, max_splits=16, block_table=None):
    dev = torch.device("cuda")
    pc = W.paged_from_packed(w, page_size, seed=seed)
    bt = pc.block_table if block_table is None else block_table
    q, kp, vp, bt_d, sl = (t.to(dev) for t in (w.q, pc.k_pages, pc.v_pages, bt, pc.seq_lens))
    ns = None if num_splits is None else torch.as_tensor(num_splits, dtype=torch.int32, device=dev)
    o, lse = attn.decode_paged(q, kp, vp, bt_d, sl, num_splits=ns, max_splits=max_splits, scale=w.scale)
    torch.cuda.synchronize()
    return np64(o), np64(lse), pc


def ref_paged(w, pc):
    return oracle.decode_attention_paged(np64(w.q), np64(pc.k_pages), np64(pc.v_pages), pc.block_table.numpy(),
                                         pc.seq_lens.numpy(), w.scale)


@pytest.mark.parametrize("lengths,Hq,Hkv,D,page", [
    ([1, 2, 15, 16, 17, 0, 1000, 257], 8, 2, 128, 16),   # block-sized pages, empty and 1-key streams
    ([4096, 1, 513, 64, 65], 32, 8, 128, 64),
    ([300, 7000, 64], 16, 1, 64, 256),                    # G = 16
    ([100, 200, 31], 6, 3, 64, 32),                       # G = 2
    ([129, 31, 256], 3, 3, 128, 128),                     # G = 1
])
def test_decode_paged_shapes(lengths, Hq, Hkv, D, page):
    w = W.random_decode(len(lengths), Hq, Hkv, D, lengths, seed=sum(lengths) + page)
    o, lse, pc = run_paged(w, page, seed=page)
    assert attn.device_status() == 0
    assert attn.last_path(2) == "decode_splitkv_paged_mma16816"
    assert np.all(np.isfinite(o))                         # no NaN pool row was read
    o_ref, lse_ref = ref_paged(w, pc)
    assert_o_bf16(o, o_ref)
    assert_lse(lse, lse_ref)


def test_decode48_paged_matches_packed_oracle():
    w = W.decode48()
    o, lse, _ = run_paged(w, 64, seed=3)
    assert attn.device_status() == 0
    o_ref, lse_ref = ref(w)                               # the same keys, packed
    assert_o_bf16(o, o_ref)
    assert_lse(lse, lse_ref)


def test_decode_paged_split_counts_change_rounding_only():
    w = W.random_decode(5, 8, 2, 128, [3000, 1500, 17, 4096, 33], seed=12)
    outs = []
    for ns in ([1] * 5, [16] * 5, [3, 7, 1, 13, 2], [64] * 5):
        o, lse, pc = run_paged(w, 32, seed=1, num_splits=ns, max_splits=64)
        assert attn.device_status() == 0
        o_ref, lse_ref = ref_paged(w, pc)
        assert_o_bf16(o, o_ref)
        assert_lse(lse, lse_ref)
        outs.append(o)
    for o in outs[1:]:
        assert max_abs(o, outs[0]) <= 2e-2


def test_decode_paged_bad_page_id_is_reported_not_read():
    # one table entry points one page past the pool: that page is never read (its keys count as
    # zeros), the device status says ATTN_ERR_INVALID_ARG, and the other streams are unaffected
    w = W.random_decode(3, 8, 2, 128, [100, 40, 70], seed=5)
    pc = W.paged_from_packed(w, 16, seed=1)
    bt = pc.block_table.clone()
    bt[1, 1] = pc.k_pages.shape[0]
    o, lse, _ = run_paged(w, 16, seed=1, block_table=bt)
    assert attn.device_status() == 1
    assert attn.device_status() == 0                      # reading clears it
    o_ref, lse_ref = ref_paged(w, pc)
    assert_o_bf16(o[[0, 2]], o_ref[[0, 2]])
    assert_lse(lse[[0, 2]], lse_ref[[0, 2]])
