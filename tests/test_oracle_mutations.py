"""Plant plausible mistakes in the oracle (on the CPU) and check that the pins
catch each one.  A pin suite that passes a broken oracle pins nothing."""
import numpy as np
import pytest

import oracle.attn as oatt
import oracle.cache as ocache
import oracle.moba as omoba
import oracle.rope as orope
from tests import test_oracle_attention as t_att
from tests import test_oracle_cache as t_cache
from tests import test_oracle_moba as t_moba
from tests import test_oracle_rope as t_rope


def _fails(fn, *args):
    with pytest.raises(AssertionError):
        fn(*args)


def _rope_variant(kind):
    def bad(x, t, h, w, pairs, base=10000.0):
        x = np.asarray(x, dtype=np.float64)
        N, H, D = x.shape
        pos = [np.asarray(t, float), np.asarray(h, float), np.asarray(w, float)]
        if kind == "swap_hw":
            pos[1], pos[2] = pos[2], pos[1]
        out = x.copy()
        for i in range(D // 2):
            axis, j = orope.axis_of_pair(i, pairs)
            if kind == "half_split":
                a, b = i, i + D // 2
            else:
                a, b = 2 * i, 2 * i + 1
            P = pairs[axis]
            freq = base ** (-(2.0 * j) / (2.0 * P)) if kind != "freq_D" else base ** (-(2.0 * j) / D)
            ang = pos[axis] * freq
            c, s = np.cos(ang)[:, None], np.sin(ang)[:, None]
            if kind == "sign":
                s = -s
            x0, x1 = x[:, :, a], x[:, :, b]
            out[:, :, a] = x0 * c - x1 * s
            out[:, :, b] = x0 * s + x1 * c
        return out
    return bad


@pytest.mark.parametrize("kind", ["sign", "swap_hw", "half_split", "freq_D"])
def test_rope_mutations_caught(monkeypatch, kind):
    monkeypatch.setattr(t_rope, "rope3d", _rope_variant(kind))
    caught = 0
    for args in t_rope._read_golden():
        try:
            t_rope.test_hand_derived_angles(*args)
        except AssertionError:
            caught += 1
    try:
        t_rope.test_axes_are_separate()
        t_rope.test_single_axis_reduces_to_textbook_rope()
    except AssertionError:
        caught += 1
    assert caught > 0


class _EvictNewest(ocache.CacheModel):
    def append(self, frames):
        slots, ev = [], []
        for f in frames:
            if self.n_sinks_filled < self.sinks:
                s = self.n_sinks_filled
                self.n_sinks_filled += 1
            elif len(self.recent) == self.window:
                old = self.recent.pop()            # planted: newest instead of oldest
                s = self.frame_slot.pop(old)
                ev.append(old)
                self.recent.append(f)
            else:
                s = min(i for i in range(self.sinks, self.sinks + self.window)
                        if self.slot_frame[i] == -1)
                self.recent.append(f)
            self.slot_frame[s] = f
            self.frame_slot[f] = s
            slots.append(s)
        return slots, ev


class _SinksEvictable(ocache.CacheModel):
    def __init__(self, sinks, window):
        super().__init__(0, sinks + window)        # planted: no pinned anchors


@pytest.mark.parametrize("bad", [_EvictNewest, _SinksEvictable])
def test_cache_mutations_caught(monkeypatch, bad):
    monkeypatch.setattr(t_cache, "CacheModel", bad)
    _fails(t_cache.test_worked_examples, "slot_map_6anchor_8window.txt", 6, 8, 4, 1508)


def test_attention_mutations_caught(monkeypatch):
    def no_norm(q, k, v, scale):
        o, lse = oatt.attention(q, k, v, scale)
        return o * 1.5, lse
    monkeypatch.setattr(t_att, "attention", no_norm)
    _fails(t_att.test_zero_query_gives_mean_and_log_n)

    def no_scale(q, k, v, scale):
        return oatt.attention(q, k, v, 1.0)
    monkeypatch.setattr(t_att, "attention", no_scale)
    _fails(t_att.test_matches_bruteforce_loops)


def test_moba_mutation_caught(monkeypatch):
    def bad_allowed(qpos, kpos, lay):
        qk, qi = omoba.block_of(qpos, lay)
        kk, ki = omoba.block_of(kpos, lay)
        c_row = (qk == 0) & (kk == 0) & (ki <= qi)
        n_row = (qk == 1) & (((kk == 0) & (ki <= qi)) | ((kk == 1) & (ki == qi)))  # planted j <= i
        b_row = (qk == 2) & (kk == 2)
        return c_row | n_row | b_row

    def bad_mask(lay):
        pos = np.arange(lay.seq_len)
        return bad_allowed(pos[:, None], pos[None, :], lay)
    monkeypatch.setattr(t_moba, "moba_mask", bad_mask)
    _fails(t_moba.test_rule_table)


# ------------------------------------------------ auxiliary frames, fp8, backward
import importlib                          # noqa: E402

oroll = importlib.import_module("oracle.rollout")   # the package also exports a function of that name
ofp8 = importlib.import_module("oracle.fp8")
obwd = importlib.import_module("oracle.moba_bwd")
from tests import test_oracle_aux as t_aux          # noqa: E402
from tests import test_oracle_fp8 as t_fp8          # noqa: E402
from tests import test_oracle_moba_bwd as t_bwd     # noqa: E402


def test_aux_keys_left_unrotated_is_caught(monkeypatch):
    """Auxiliary K used raw although positions were given: the key-duplication pin fails."""
    real = oroll.rope3d
    calls = {"n": 0}

    def skip_aux_rotation(x, t, h, w, pairs, base=10000.0):
        # the rollout rotates Q, K of the chunk (2 calls) and then the auxiliary K
        calls["n"] += 1
        if calls["n"] % 3 == 0:
            return np.asarray(x, dtype=np.float64)
        return real(x, t, h, w, pairs, base)
    monkeypatch.setattr(oroll, "rope3d", skip_aux_rotation)
    _fails(t_aux.test_copies_of_every_visible_frame_double_each_key)


def test_fp8_ties_away_from_zero_is_caught(monkeypatch):
    real_pos = ofp8._POS

    def ties_away(x):
        x = np.asarray(x, dtype=np.float64)
        a = np.abs(x)
        i = np.clip(np.searchsorted(real_pos, a, side="left"), 1, real_pos.size - 1)
        lo, hi = real_pos[i - 1], real_pos[i]
        r = np.where(hi - a <= a - lo, hi, lo)            # ties up instead of to even
        r = np.where(a >= real_pos[-1], 448.0, r)
        return np.copysign(np.where(a <= 0, 0.0, r), x)
    monkeypatch.setattr(ofp8, "e4m3_round", ties_away)
    _fails(t_fp8.test_ties_go_to_the_even_mantissa)


def test_fp8_one_scale_per_tensor_is_caught(monkeypatch):
    """One amax for the whole tensor (per head) instead of one per 128-row block."""
    def per_tensor(x, rows=128):
        x = np.asarray(x, dtype=np.float32)
        nb = (x.shape[0] + rows - 1) // rows
        amax = np.abs(x).max(axis=(0, 2)).astype(np.float32)
        codes = np.zeros(x.shape)
        for h in range(x.shape[1]):
            inv = np.float32(448.0) / amax[h]
            codes[:, h] = ofp8.e4m3_round((x[:, h] * inv).astype(np.float32))
        return codes, np.tile(amax / np.float32(448.0), (nb, 1))
    monkeypatch.setattr(ofp8, "quantize_blocks", per_tensor)
    _fails(t_fp8.test_block_quantization)


def test_bwd_missing_scale_on_dk_is_caught(monkeypatch):
    real = obwd.attention_bwd_masked

    def no_scale_dk(q, k, v, do, allowed, scale):
        dq, dk, dv = real(q, k, v, do, allowed, scale)
        return dq, dk / scale, dv
    monkeypatch.setattr(obwd, "attention_bwd_masked", no_scale_dk)
    _fails(t_bwd.test_matches_central_finite_differences, 2, 3, 1)
