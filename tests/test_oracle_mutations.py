"""Plant plausible mistakes in the oracle (on the CPU) and check that the pins
catch every one of them."""
import numpy as np
import pytest

import oracle_pins
from oracle import hisa_oracle as ho
from oracle import ofp8
from oracle import sparse_attention as sa


def _no_relu(q_t, w_t, keys):
    return (np.asarray(keys, np.float64) @ np.asarray(q_t, np.float64).T) @ np.asarray(w_t, np.float64)


def _heads_swapped(q_t, w_t, keys):
    q = np.asarray(q_t, np.float64)[::-1]
    return np.maximum(np.asarray(keys, np.float64) @ q.T, 0) @ np.asarray(w_t, np.float64)


def _ties_high(scores, count):
    scores = np.asarray(scores, np.float64)
    n = len(scores)
    order = np.lexsort((-np.arange(n), -scores))
    return order[:min(count, n)]


def _current_block_late(n_t, block):
    return n_t // block if n_t > 0 else -1


def _blocks_unforced(q_t, w_t, kpool, n_t, block, top_m):
    c = ho.current_block(n_t, block)
    if c < 0:
        return np.zeros(0, np.int64)
    s = ho.indexer_scores(q_t, w_t, kpool[:c + 1])
    return np.sort(ho.top_by_score(s, top_m)).astype(np.int64)


def _block_sums(keys, block):
    keys = np.asarray(keys, np.float64)
    nb = -(-keys.shape[0] // block)
    return np.stack([keys[b * block:(b + 1) * block].sum(axis=0) for b in range(nb)])


def _mean_of_relu_blocks(q_t, w_t, kpool, n_t, block, top_m):
    # scores blocks by pooling after the ReLU (needs the raw keys; emulate on kpool rows)
    c = ho.current_block(n_t, block)
    if c < 0:
        return np.zeros(0, np.int64)
    if c + 1 <= top_m:
        return np.arange(c + 1, dtype=np.int64)
    s = np.abs(np.asarray(kpool[:c], np.float64) @ np.asarray(q_t, np.float64).T) @ np.asarray(w_t)
    kept = ho.top_by_score(s, top_m - 1)
    return np.sort(np.concatenate([kept, [c]])).astype(np.int64)


def _cand_leaky(blocks, n_t, block):
    parts = [np.arange(b * block, min((b + 1) * block, n_t + 1)) for b in sorted(blocks)]
    return np.concatenate(parts).astype(np.int64) if parts else np.zeros(0, np.int64)


def _e4m3_half_away(x):
    x = np.asarray(x, np.float64)
    nudged = x + np.sign(x) * np.abs(x) * 1e-9
    return _orig_e4m3(nudged)


def _bf16_via_fp32(x):
    return _orig_bf16(np.asarray(x, np.float64).astype(np.float32).astype(np.float64))


def _superblock_leaky(superblocks, c_t, group):
    # also takes the current block and the partial blocks after it
    parts = [np.arange(u * group, (u + 1) * group) for u in sorted(superblocks)]
    return np.concatenate(parts).astype(np.int64) if parts else np.zeros(0, np.int64)


def _second_level_unforced(q_t, w_t, kpool, cands, c_t, top_m):
    if c_t < 0 or len(cands) == 0:
        return np.zeros(0, np.int64)
    s = ho.indexer_scores(q_t, w_t, kpool[cands])
    return np.sort(cands[ho.top_by_score(s, top_m)]).astype(np.int64)


def _padding_as_position(idx_row, num_keys=None):
    return np.unique(np.asarray(idx_row, np.int64))          # -1 reads the last key


def _out_of_range_kept(idx_row, num_keys=None):
    r = np.asarray(idx_row, np.int64)
    return np.unique(r[r >= 0])                               # entries past the keys are not dropped


def _repeats_counted(idx_row, num_keys=None):
    r = np.asarray(idx_row, np.int64)
    return np.sort(r[(r >= 0) & (r < (num_keys if num_keys is not None else np.iinfo(np.int64).max))])                                 # a repeated index weighs twice


_orig_attn = sa.sparse_attention_query


def _softmax_over_heads(q_t, keys, values, idx_row, scale):
    s = sa.selected_positions(idx_row)
    if s.size == 0:
        return _orig_attn(q_t, keys, values, idx_row, scale)
    logits = scale * (np.asarray(q_t, np.float64) @ np.asarray(keys, np.float64)[s].T)
    e = np.exp(logits - logits.max(axis=0, keepdims=True))
    p = e / e.sum(axis=0, keepdims=True)
    return p @ np.asarray(values, np.float64)[s], np.log(np.exp(logits).sum(axis=1))


def _scale_dropped(q_t, keys, values, idx_row, scale):
    return _orig_attn(q_t, keys, values, idx_row, 1.0)


def _lse_without_max(q_t, keys, values, idx_row, scale):
    o, lse = _orig_attn(q_t, keys, values, idx_row, scale)
    s = sa.selected_positions(idx_row)
    if s.size:
        lg = scale * (np.asarray(q_t, np.float64) @ np.asarray(keys, np.float64)[s].T)
        lse = lse - lg.max(axis=1)
    return o, lse


def _pool_e4m3_ratio_in_fp64(codes, scale, block):
    # scale and quotient kept in float64: no fp32 decision
    means = ho.block_means(ho.dequantize_e4m3_rows(codes, scale), block)
    amax = np.abs(means).max(axis=1)
    s = np.where(amax > 0, amax / 448.0, 1.0)
    return ofp8.e4m3_encode(means / s[:, None]), s.astype(np.float32)


def _pool_e4m3_mean_unrounded(codes, scale, block):
    # fp32 scale, but the float64 mean is divided before any fp32 rounding
    means = ho.block_means(ho.dequantize_e4m3_rows(codes, scale), block)
    amax = np.abs(means.astype(np.float32)).max(axis=1)
    s = np.where(amax > 0, amax / np.float32(448.0), np.float32(1.0)).astype(np.float32)
    return ofp8.e4m3_encode((means / s[:, None].astype(np.float64)).astype(np.float32)), s


def _pool_e4m3_scale_from_keys(codes, scale, block):
    # block scale from the absmax of the block's dequantised keys, not of their mean
    deq = ho.dequantize_e4m3_rows(codes, scale)
    means = ho.block_means(deq, block).astype(np.float32)
    nb = means.shape[0]
    amax = np.array([np.abs(deq[b * block:(b + 1) * block]).max() for b in range(nb)], np.float32)
    s = np.where(amax > 0, amax / np.float32(448.0), np.float32(1.0)).astype(np.float32)
    return ofp8.e4m3_encode((means / s[:, None]).astype(np.float32)), s


def _q_scale_per_head(q):
    q = np.asarray(q)
    Qn, H, d = q.shape
    codes, scale = ho.quantize_e4m3_rows(q.reshape(Qn * H, d).astype(np.float32))
    return codes.reshape(Qn, H, d), scale.reshape(Qn, H).max(axis=1)


_orig_e4m3 = ofp8.e4m3_encode
_orig_bf16 = ofp8.bf16_round

MUTATIONS = {
    "relu_dropped": [(ho, "indexer_scores", _no_relu)],
    "weights_on_wrong_heads": [(ho, "indexer_scores", _heads_swapped)],
    "ties_to_higher_index": [(ho, "top_by_score", _ties_high)],
    "current_block_off_by_one": [(ho, "current_block", _current_block_late)],
    "current_block_not_forced": [(ho, "select_blocks", _blocks_unforced)],
    "pool_sum_not_mean": [(ho, "block_means", _block_sums)],
    "block_score_abs": [(ho, "select_blocks", _mean_of_relu_blocks)],
    "causal_leak": [(ho, "candidate_keys", _cand_leaky)],
    "three_levels_partial_blocks": [(ho, "candidate_blocks", _superblock_leaky)],
    "three_levels_current_not_forced": [(ho, "select_blocks_among", _second_level_unforced)],
    "e4m3_ties_away": [(ofp8, "e4m3_encode", _e4m3_half_away), (ho, "e4m3_encode", _e4m3_half_away)],
    "bf16_double_rounding": [(ofp8, "bf16_round", _bf16_via_fp32), (ho, "bf16_round", _bf16_via_fp32)],
    "e4m3_pool_quotient_in_fp64": [(ho, "pool_blocks_e4m3", _pool_e4m3_ratio_in_fp64)],
    "e4m3_pool_mean_not_rounded_to_fp32": [(ho, "pool_blocks_e4m3", _pool_e4m3_mean_unrounded)],
    "e4m3_pool_scale_from_keys": [(ho, "pool_blocks_e4m3", _pool_e4m3_scale_from_keys)],
    "e4m3_q_scale_per_head": [(ho, "quantize_q_tokens", _q_scale_per_head)],
    "attention_padding_as_position": [(sa, "selected_positions", _padding_as_position)],
    "attention_repeats_counted": [(sa, "selected_positions", _repeats_counted)],
    "attention_out_of_range_kept": [(sa, "selected_positions", _out_of_range_kept)],
    "attention_softmax_over_heads": [(sa, "sparse_attention_query", _softmax_over_heads)],
    "attention_scale_dropped": [(sa, "sparse_attention_query", _scale_dropped)],
    "attention_lse_without_max": [(sa, "sparse_attention_query", _lse_without_max)],
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_mutation_is_caught(name, monkeypatch):
    for mod, attr, fn in MUTATIONS[name]:
        monkeypatch.setattr(mod, attr, fn)
    caught = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin()
        except Exception:       # an assertion, or the mistake breaking a shape
            caught.append(pin.__name__)
    assert caught, f"no pin catches the planted mistake {name!r}"
