"""The benchmark's algorithmic byte counts (the roofline numerators) on CPU.

Per (sequence, kv-head) a sparse step reads the packed int4 keys (D/2 = 64 B per
token) and one bf16 scale row per block (2 D = 256 B) in the scan, and bf16 K
and V (4 D = 512 B per token) of the kept tokens; the thumbnail format reads
32 B of thumbnails per token in the scan and 128 B of residuals + 256 B of V
per kept token.  The expected values below are those products written out for
each workload's full-length shape.
"""
import numpy as np
import pytest

import bench
import ffd_workloads as fw

# name: (scan bytes, dense K/V bytes) at full lengths
FULL = {
    "tiny": (278_528, 2_097_152),
    "llama": (71_303_168, 536_870_912),
    "long128k": (71_303_168, 536_870_912),
    "max256k": (138_412_032, 1_073_741_824),
}


def _full(name):
    w = fw.WORKLOADS[name]
    lengths = np.full(w.batch, w.context, np.int64)
    return w, lengths, int(lengths.sum()) * w.num_kv_heads


@pytest.mark.parametrize("name", sorted(FULL))
def test_int4_scan_and_kv_bytes(name):
    w, lengths, tokens = _full(name)
    scan, dense_kv = FULL[name]
    a = bench.algorithmic_bytes(w, lengths, tokens, dense=False)
    assert a["scan"] == scan
    assert a["kv"] == dense_kv
    d = bench.algorithmic_bytes(w, lengths, tokens, dense=True)
    assert d["scan"] == 0 and d["kv"] == dense_kv
    assert a["total"] - d["total"] == scan


@pytest.mark.parametrize("name", sorted(FULL))
def test_thumbnail_bytes(name):
    w, lengths, tokens = _full(name)
    nb = w.context // w.block_size
    thumb_scan = w.batch * w.num_kv_heads * (w.context * 32 + nb * 256)
    a = bench.algorithmic_bytes_tr(w, lengths, tokens, dense=False)
    assert a["scan"] == thumb_scan
    assert a["kv"] == tokens * (128 + 256)
    # dense: the computer reads the thumbnails and scales the scan would have
    d = bench.algorithmic_bytes_tr(w, lengths, tokens, dense=True)
    assert d["scan"] == 0 and d["kv"] == tokens * (128 + 256) + thumb_scan
    assert a["total"] == d["total"]


def test_fixed_terms_at_128k():
    # one re-quantised block per kv-head (64 K rows read, packed rows and a
    # scale row written), q and out (bf16), the mask words, and the split
    # partials (32 splits x 4 heads x 130 floats, written and read)
    w, lengths, tokens = _full("long128k")
    a = bench.algorithmic_bytes(w, lengths, tokens, dense=False)
    assert a["requant"] == 8 * (64 * 256 + 64 * 64 + 256)
    assert a["q_out_mask"] == 2 * 32 * 128 * 2 + 8 * 64 * 4
    assert a["partials"] == 8 * 32 * 4 * 130 * 4 * 2
    t = bench.algorithmic_bytes_tr(w, lengths, tokens, dense=False)
    assert t["requant"] == 8 * (64 * 256 + 64 * (32 + 128) + 256)


def test_kept_tokens_from_mask_counts_partial_blocks():
    # the last block of a sequence counts only its valid tokens
    w = fw.scaled_workload(fw.WORKLOADS["tiny"], batch=2, capacity=4096)
    T, nblk = w.block_size, 4096 // 64
    lengths = np.array([T * 3 + 5, T * 10], np.int32)
    mask = np.zeros((2, 1, nblk // 32), np.uint32)
    mask[0, 0, 0] = 0b1011  # blocks 0, 1, 3 (block 3 holds 5 tokens)
    mask[1, 0, 0] = 1 << 9  # block 9, full
    kept_blocks, valid_blocks, kept_tok = bench.kept_tokens_from_mask(w, lengths, mask)
    assert (kept_blocks, valid_blocks, kept_tok) == (4, 4 + 10, 2 * T + 5 + T)
