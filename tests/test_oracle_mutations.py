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
