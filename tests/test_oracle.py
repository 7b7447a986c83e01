"""The oracle against its pins, and the pins against planted mistakes."""
import numpy as np
import pytest

import oracle.kv_decode as kv
from tests import oracle_pins as pins


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda f: f.__name__)
def test_oracle_pin(pin):
    pin(kv)


# --- planted mistakes: each mutation of the oracle must fail at least one pin.
def _rope_interleaved(x, positions, base, interleaved=False, rotary_dim=0):
    """Always pairs (2j, 2j + 1), whatever the layout asked for."""
    return _orig_rope(x, positions, base, True, rotary_dim)


def _rope_wrong_sign(x, positions, base, interleaved=False, rotary_dim=0):
    return _orig_rope(x, -np.asarray(positions), base, interleaved, rotary_dim)


def _rope_ignores_layout(x, positions, base, interleaved=False, rotary_dim=0):
    return _orig_rope(x, positions, base)


def _rope_partial_full_width_freq(x, positions, base, interleaved=False, rotary_dim=0):
    """Partial rotation with theta_j = base^(-2j/D) instead of base^(-2j/r)."""
    x = np.asarray(x, np.float64)
    D = x.shape[-1]
    r = rotary_dim or D
    if r == D:
        return _orig_rope(x, positions, base, interleaved)
    scaled_base = float(base) ** (r / D)     # base'^(-2j/r) = base^(-2j/D)
    out = x.copy()
    out[..., :r] = _orig_rope(x[..., :r], positions, scaled_base, interleaved)
    return out


def _rope_partial_rotates_all(x, positions, base, interleaved=False, rotary_dim=0):
    """Rotates all D elements with the rotary-width frequencies of the first r."""
    x = np.asarray(x, np.float64)
    D = x.shape[-1]
    r = rotary_dim or D
    out = _orig_rope(x, positions, base, interleaved, r)
    if r < D:
        out[..., r:] = _orig_rope(x[..., r:], positions, base, interleaved)
    return out


def _inv_freq_off(head_dim, base):
    j = np.arange(head_dim // 2, dtype=np.float64)
    return np.power(float(base), -2.0 * (j + 1) / head_dim)


def _attend_no_scale(q_rows, K, V, scale, visible):
    return _orig_attend(q_rows, K, V, 1.0, visible)


def _attend_off_by_one(q_rows, K, V, scale, visible):
    return _orig_attend(q_rows, K, V, scale, np.maximum(np.asarray(visible) - 1, 1))


def _attend_transposed(q_rows, K, V, scale, visible):
    return _orig_attend(q_rows, V, K, scale, visible)


def _bf16_truncate(x):
    x = np.asarray(x, np.float64)
    out = x.copy()
    sel = np.isfinite(x) & (x != 0)
    v = x[sel]
    _, e = np.frexp(v)
    sp = np.maximum(e - 8, -133)
    out[sel] = np.ldexp(np.trunc(np.ldexp(v, -sp)), sp)
    return out


def _gather_mod_heads(cache, b, h, n, block_table=None):
    return _orig_gather(cache, b, (h + 1) % cache.shape[1], n, block_table)


def _merge_plain_mean(o_parts, lse_parts):
    o = np.asarray(o_parts, np.float64)
    live = np.isfinite(np.asarray(lse_parts))
    return (o * live[..., None]).sum(0) / np.maximum(live.sum(0), 1)[..., None]


def _attend_partial_natural_log(q_rows, K, V, scale, visible):
    o, lse = _orig_attend_partial(q_rows, K, V, scale, visible)
    return o, lse * kv.LN2


def _shard_no_offset(q_rot, k_local, v_local, seq_lens, shard_start, shard_lens, scale,
                     block_table=None):
    return _orig_shard(q_rot, k_local, v_local, seq_lens, np.zeros_like(shard_start), shard_lens,
                       scale, block_table)


def _append_cow_skipped(*args, **kw):
    kw.pop("cow_src", None)
    return _orig_append(*args, **kw)


def _max_diff_signed(a, b):
    """max (a - b) instead of max |a - b|."""
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    return float(np.max(a - b)) if a.size else 0.0


def _max_diff_mean(a, b):
    """mean |a - b| instead of the max."""
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    return float(np.mean(np.abs(a - b))) if a.size else 0.0


def _max_diff_skips_nan(a, b):
    """NaN-skipping max: a poisoned element would pass every check."""
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    d = np.abs(a - b)
    return float(np.nanmax(d)) if a.size and not np.isnan(d).all() else 0.0


def _max_diff_broadcasts(a, b):
    """No shape check: mismatched arrays are broadcast against each other."""
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    return float(np.max(np.abs(a - b))) if a.size else 0.0


def _max_diff_first_row(a, b):
    """Compares only the first element along the leading axis."""
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    if a.shape != b.shape:
        raise ValueError("shapes differ")
    return float(np.max(np.abs(a[:1] - b[:1]))) if a.size else 0.0


_orig_append = kv.append_rope
_orig_attend = kv.attend
_orig_attend_partial = kv.attend_partial
_orig_shard = kv.decode_attention_shard
_orig_rope = kv.rope
_orig_gather = kv.gather_tokens

MUTANTS = {
    "rope_interleaved_pairs": ("rope", _rope_interleaved),
    "rope_wrong_sign": ("rope", _rope_wrong_sign),
    "rope_ignores_layout": ("rope", _rope_ignores_layout),
    "rope_partial_full_width_freq": ("rope", _rope_partial_full_width_freq),
    "rope_partial_rotates_all": ("rope", _rope_partial_rotates_all),
    "rope_freq_index_off": ("rope_inv_freq", _inv_freq_off),
    "attend_drops_scale": ("attend", _attend_no_scale),
    "attend_mask_off_by_one": ("attend", _attend_off_by_one),
    "attend_k_v_swapped": ("attend", _attend_transposed),
    "bf16_truncates": ("bf16_round", _bf16_truncate),
    "wrong_kv_head": ("gather_tokens", _gather_mod_heads),
    "merge_ignores_lse": ("merge_partials", _merge_plain_mean),
    "partial_lse_natural_log": ("attend_partial", _attend_partial_natural_log),
    "shard_mask_ignores_offset": ("decode_attention_shard", _shard_no_offset),
    "copy_on_write_skipped": ("append_rope", _append_cow_skipped),
    "max_abs_diff_signed": ("max_abs_diff", _max_diff_signed),
    "max_abs_diff_mean": ("max_abs_diff", _max_diff_mean),
    "max_abs_diff_skips_nan": ("max_abs_diff", _max_diff_skips_nan),
    "max_abs_diff_broadcasts": ("max_abs_diff", _max_diff_broadcasts),
    "max_abs_diff_first_row": ("max_abs_diff", _max_diff_first_row),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name, monkeypatch):
    attr, fn = MUTANTS[name]
    monkeypatch.setattr(kv, attr, fn)
    failed = []
    for pin in pins.ALL_PINS:
        try:
            pin(kv)
        except (AssertionError, ValueError, IndexError):
            failed.append(pin.__name__)
    assert failed, f"no pin caught the planted mistake {name}"
