"""Planted mistakes in the oracle, one per entry, to check that its pins catch
them.  Each entry patches the oracle modules in place; ``conftest.py`` applies
the one named by the environment variable FT_ORACLE_MUTANT (only ever set by
``test_oracle_mutants.py`` for a child pytest process).  Every mistake is a
plausible slip when writing the oracle from its definitions: a wrong table
entry, nibble or byte order, a rounding rule, a tie rule, a summation order, a
swapped operand, a dropped term, a wrong recency rule."""
from __future__ import annotations

import math

import numpy as np

from oracle import formats, fp4, layer, lru, routing


# ---------------------------------------------------------------------------
# e2m1 / UE8M0 decoding and the blob's storage index
# ---------------------------------------------------------------------------

def e2m1_magnitude():
    fp4.E2M1_TABLE[5], fp4.E2M1_TABLE[13] = 2.5, -2.5          # 3.0 decoded as 2.5


def e2m1_negative_zero():
    fp4.E2M1_TABLE[8] = 0.0                                     # code 8 as +0


def ue8m0_bias():
    fp4.UE8M0_TABLE[:255] = np.ldexp(1.0, np.arange(255) - 126)


def nibble_order():
    orig = fp4.dequant_matrix

    def f(blob, which, hidden, inter):
        off = fp4.layout(hidden, inter)
        rows, K = (inter, hidden) if which in ("wg", "wu") else (hidden, inter)
        b = np.array(blob, dtype=np.uint8, copy=True)
        seg = b[off[which]: off[which] + rows * K // 2]
        b[off[which]: off[which] + rows * K // 2] = (seg >> 4) | (seg << 4)   # element 2i read from the high nibble
        return orig(b, which, hidden, inter)
    fp4.dequant_matrix = f


def pack_high_nibble_first():
    fp4.pack_codes = lambda codes: ((codes[:, 0::2] << 4) | codes[:, 1::2]).astype(np.uint8)


def dequant_rows_scales_tiled():
    # np.tile where np.repeat belongs: element k takes block k mod (K/32)'s scale
    fp4.dequant_rows = lambda codes, scales: fp4.E2M1_TABLE[codes] * np.tile(fp4.UE8M0_TABLE[scales], (1, 32))


def bf16_decode_low_half():
    fp4.bf16_to_f64 = lambda bits: (np.asarray(bits, dtype=np.uint16).astype(np.uint32)).view(np.float32).astype(
        np.float64)


def _scale_index(word_of, byte_of):
    def f(row, kblock, n_kblocks):
        atoms_k = -(-int(n_kblocks) // 4)
        atom = (row // 128) * atoms_k + kblock // 4
        return atom * 512 + word_of(row, kblock) + byte_of(row, kblock)
    return f


def scale_atom_row_major():
    fp4.scale_index = _scale_index(lambda r, kb: (r % 128) * 4, lambda r, kb: kb % 4)


def scale_word_byte_swapped():
    fp4.scale_index = _scale_index(lambda r, kb: (r % 32) * 16 + (kb % 4) * 4, lambda r, kb: (r % 128) // 32)


# ---------------------------------------------------------------------------
# OCP MX quantiser and bf16 rounding
# ---------------------------------------------------------------------------

def _rows_via_blocks():
    """quantize_rows through the (patched) scalar quantize_block, so both forms
    carry the same mistake."""
    def f(v):
        v = np.asarray(v, dtype=np.float64)
        R, K = v.shape
        codes = np.empty((R, K), np.uint8)
        sc = np.empty((R, K // 32), np.uint8)
        for r in range(R):
            for b in range(K // 32):
                codes[r, 32 * b:32 * b + 32], sc[r, b] = fp4.quantize_block(v[r, 32 * b:32 * b + 32])
        return codes, sc
    fp4.quantize_rows = f

    def g(a):
        a = np.asarray(a, dtype=np.float64)
        return np.vectorize(fp4._round_to_grid, otypes=[np.uint8])(a) if a.size else a.astype(np.uint8)
    fp4.round_to_grid_vec = g


def quant_emax_one():
    fp4.block_scale_byte = lambda amax: 0 if amax == 0.0 else int(min(max(math.frexp(amax)[1] - 1 + 127 - 1, 0), 254))
    _rows_via_blocks()


def quant_ties_away():
    def r(a):
        if a >= 6.0:
            return 7
        best = None
        for c, gv in enumerate(fp4.E2M1_GRID):
            d = abs(a - gv)
            if best is None or d <= best[0]:          # the larger code wins a tie
                best = (d, c)
        return best[1]
    fp4._round_to_grid = r
    _rows_via_blocks()


def quant_sign_of_zero():
    orig = fp4.quantize_block

    def f(v):
        codes, e = orig(v)
        return np.where(codes == 8, 0, codes).astype(np.uint8), e   # -0 stored as +0
    fp4.quantize_block = f
    _rows_via_blocks()


def _bf16_rounding(mode):
    def bits(v):
        v = np.asarray(v, dtype=np.float64)
        if mode == "via_fp32":
            v = v.astype(np.float32).astype(np.float64)       # double rounding
        a = np.abs(v)
        _, ex = np.frexp(np.where(a == 0.0, 1.0, a))
        ue = np.maximum(ex - 1, -126) - 7
        q = np.ldexp(a, -ue)
        r = np.floor(q)
        frac = q - r
        if mode == "away":
            r = r + (frac >= 0.5)
        elif mode == "via_fp32":
            r = r + ((frac > 0.5) | ((frac == 0.5) & (np.fmod(r, 2.0) == 1.0)))
        val = np.ldexp(r, ue)                                   # mode "truncate": r as is
        out = (val.astype(np.float32).view(np.uint32) >> np.uint32(16)).astype(np.uint32)
        out = np.where(val >= 2.0 ** 128, 0x7F80, out)
        out = np.where(a == 0.0, 0, out)
        out = out | np.where(np.signbit(v), 0x8000, 0)
        out = np.where(np.isnan(v), 0x7FC0, out)
        return out.astype(np.uint16)
    fp4.round_bf16 = bits
    fp4.round_bf16_scalar = lambda x: int(bits(np.array([float(x)]))[0])


def bf16_ties_away():
    _bf16_rounding("away")


def bf16_truncate():
    _bf16_rounding("truncate")


def bf16_via_fp32():
    _bf16_rounding("via_fp32")


# ---------------------------------------------------------------------------
# routing
# ---------------------------------------------------------------------------

def topk_ties_to_higher_id():
    orig = routing.topk

    def f(logits, k):
        lg = np.asarray(logits, dtype=np.float32)
        ids, bad = orig(lg[:, ::-1], k)
        return (lg.shape[1] - 1 - ids).astype(np.int32), bad
    routing.topk = f


def topk_nan_on_top():
    orig = routing.topk

    def f(logits, k):
        lg = np.asarray(logits, dtype=np.float32)
        return orig(np.where(np.isnan(lg), np.float32(np.inf), lg), k)
    routing.topk = f


def weights_not_renormalised():
    orig = routing.softmax_weights
    routing.softmax_weights = lambda logits, ids, renorm=True: orig(logits, ids, False)


def weights_reversed():
    orig = routing.softmax_weights
    routing.softmax_weights = lambda logits, ids, renorm=True: orig(logits, ids, renorm)[:, ::-1].copy()


def _logits(part_of_k, dtype=np.float64):
    def f(x, wr):
        x = np.asarray(x, dtype=np.float64)
        wr = np.asarray(wr, dtype=np.float32).astype(np.float64)
        T, H = x.shape
        E = wr.shape[0]
        out = np.empty((T, E), np.float32)
        for t in range(T):
            prod = (wr * x[t][None, :]).astype(dtype)
            part = np.zeros((E, 32), dtype)
            for kk in range(H):
                p = part_of_k(kk)
                part[:, p] = part[:, p] + prod[:, kk]
            for d in (16, 8, 4, 2, 1):
                part = part + part[:, np.arange(32) ^ d]
            out[t] = part[:, 0].astype(np.float32)
        return out
    return f


def logits_lane_of_element():
    routing.router_logits = _logits(lambda kk: kk % 32)             # k mod 32 instead of (k div 4) mod 32


def logits_fp32_partials():
    routing.router_logits = _logits(lambda kk: (kk // 4) % 32, np.float32)


def logits_left_to_right():
    def f(x, wr):
        x = np.asarray(x, dtype=np.float64)
        wr = np.asarray(wr, dtype=np.float32).astype(np.float64)
        return np.cumsum(wr[None, :, :] * x[:, None, :], axis=2)[:, :, -1].astype(np.float32)
    routing.router_logits = f


def permutation_unstable():
    orig = routing.permutation

    def f(ids, E):
        offs, perm, inv = orig(ids, E)
        perm = perm.copy()
        for e in range(E):
            perm[offs[e]:offs[e + 1]] = perm[offs[e]:offs[e + 1]][::-1]
        inv = np.empty_like(perm)
        inv[perm] = np.arange(perm.size, dtype=np.int32)
        return offs, perm, inv
    routing.permutation = f


def offsets_inclusive():
    orig = routing.permutation

    def f(ids, E):
        offs, perm, inv = orig(ids, E)
        return np.concatenate([offs[1:], offs[-1:]]).astype(np.int32), perm, inv
    routing.permutation = f


# ---------------------------------------------------------------------------
# expert FFN and combine
# ---------------------------------------------------------------------------

def silu_sign():
    layer.silu = lambda z: z / (1.0 + np.exp(z))


def _ffn(swap=False, quant_x=True, quant_h=True):
    def f(blob, hidden, inter, x, mxfp4=False, weights="mxfp4"):
        wg = formats.weight_matrix(blob, "wg", hidden, inter, weights)
        wu = formats.weight_matrix(blob, "wu", hidden, inter, weights)
        wd = formats.weight_matrix(blob, "wd", hidden, inter, weights)
        x = np.asarray(x, dtype=np.float64)
        if mxfp4 and quant_x:
            x = fp4.dequant_rows(*fp4.quantize_rows(x))
        g, u = x @ wg.T, x @ wu.T
        h = layer.silu(u) * g if swap else layer.silu(g) * u
        if mxfp4 and quant_h:
            h = fp4.dequant_rows(*fp4.quantize_rows(h))
        return h @ wd.T
    layer.expert_ffn = f


def gate_up_swapped():
    _ffn(swap=True)


def mxfp4_x_not_quantised():
    _ffn(quant_x=False)


def mxfp4_h_not_quantised():
    _ffn(quant_h=False)


def shared_expert_dropped():
    orig = layer.moe_layer

    def f(*a, **kw):
        kw["shared_blob"] = None
        return orig(*a, **kw)
    layer.moe_layer = f


# ---------------------------------------------------------------------------
# BF16 and NVFP4 expert formats
# ---------------------------------------------------------------------------

def e4m3_bias():
    formats.E4M3_TABLE[:] = [math.nan if (b & 0x7F) == 0x7F else
                             (-1.0 if b & 0x80 else 1.0) * (math.ldexp((b & 7) / 8.0, -5) if (b >> 3) & 15 == 0
                                                           else math.ldexp(1.0 + (b & 7) / 8.0, ((b >> 3) & 15) - 6))
                             for b in range(256)]


def e4m3_subnormal_as_normal():
    for b in range(256):
        if (b >> 3) & 15 == 0:
            formats.E4M3_TABLE[b] = (-1.0 if b & 0x80 else 1.0) * math.ldexp(1.0 + (b & 7) / 8.0, -7)


def _nvfp4(block=16, use_ts=True, ts_order=("wg", "wu", "wd")):
    def f(blob, which, hidden, inter):
        off = formats.nvfp4_layout(hidden, inter)
        rows, K = (inter, hidden) if which in ("wg", "wu") else (hidden, inter)
        blob = np.asarray(blob, dtype=np.uint8)
        codes = blob[off[which]: off[which] + rows * K // 2].reshape(rows, K // 2)
        elem = np.empty((rows, K), dtype=np.uint8)
        elem[:, 0::2] = codes & 0x0F
        elem[:, 1::2] = codes >> 4
        nb = K // block
        r = np.arange(rows, dtype=np.int64)[:, None]
        b = np.arange(nb, dtype=np.int64)[None, :]
        sc = formats.E4M3_TABLE[blob[off[which + "_sf"] + fp4.scale_index(r, b, nb)]]
        t = blob[off["tensor_scales"]: off["tensor_scales"] + 12].copy().view("<f4").astype(np.float64)
        ts = float(t[ts_order.index(which)]) if use_ts else 1.0
        return fp4.E2M1_TABLE[elem] * np.repeat(sc, block, axis=1) * ts
    formats.nvfp4_matrix = f


def nvfp4_blocks_of_32():
    _nvfp4(block=32)


def nvfp4_matrix_scale_dropped():
    _nvfp4(use_ts=False)


def nvfp4_matrix_scales_rotated():
    _nvfp4(ts_order=("wu", "wd", "wg"))


def _nvfp4_act(block=16, tensor_scale=True, ties_up=False):
    """The NVFP4 activation quantiser with one slip."""
    def q(v, s=None):
        v32 = np.asarray(v, dtype=np.float32)
        R, K = v32.shape
        if s is None:
            s = formats.nvfp4_global_scale(np.abs(v32).max() if v32.size else 0.0)
        s = np.float32(s) if tensor_scale else np.float32(1.0 if np.float32(s) != 0 else 0.0)
        blocks = v32.reshape(R, K // block, block)
        if s == 0:
            return np.zeros((R, K), np.uint8), np.zeros((R, K // 16), np.uint8), s
        with np.errstate(all="ignore"):
            g = np.float32(np.float32(1.0) / np.float32(s * np.float32(6.0)))
            b = (np.abs(blocks).max(axis=-1) * g).astype(np.float32)
            e = formats.e4m3_round_vec(b)
            if ties_up:  # ties to the larger byte
                pos = formats.E4M3_TABLE[:0x7F]
                hi = np.clip(np.searchsorted(pos, b, side="left"), 0, 0x7E)
                tie = (hi > 0) & (np.abs(pos[hi] - b) == np.abs(b - pos[np.clip(hi - 1, 0, 0x7E)]))
                e = np.where(tie & (b < 448), hi, e).astype(np.uint8)
            dq = (formats.E4M3_TABLE[e].astype(np.float32) * s).astype(np.float32)
            r = (np.float32(1.0) / np.where(dq > 0, dq, np.float32(1.0))).astype(np.float32)
            qv = (blocks * r[..., None]).astype(np.float32)
        mag = fp4.round_to_grid_vec(np.abs(qv).astype(np.float64))
        codes = np.where((dq > 0)[..., None], mag | np.where(np.signbit(qv), 8, 0), 0).astype(np.uint8).reshape(R, K)
        e = np.repeat(e, 16 // block, axis=1) if block < 16 else np.repeat(e, block // 16, axis=1)
        return codes, e.astype(np.uint8), s
    formats.nvfp4_quantize_rows = q


def nvfp4_act_blocks_of_32():
    _nvfp4_act(block=32)


def nvfp4_act_tensor_scale_dropped():
    _nvfp4_act(tensor_scale=False)


def nvfp4_act_scale_ties_up():
    _nvfp4_act(ties_up=True)


def nvfp4_act_h_scale_per_expert():
    def f(x, groups, hidden, inter):
        cx, bx, sx = formats.nvfp4_quantize_rows(x)
        xq = formats.nvfp4_dequant_rows(cx, bx, sx)
        ys = []
        for blob, rows in groups:
            wg = formats.weight_matrix(blob, "wg", hidden, inter, "nvfp4")
            wu = formats.weight_matrix(blob, "wu", hidden, inter, "nvfp4")
            wd = formats.weight_matrix(blob, "wd", hidden, inter, "nvfp4")
            h = layer.silu(xq[rows] @ wg.T) * (xq[rows] @ wu.T)
            ys.append(formats.nvfp4_dequant_rows(*formats.nvfp4_quantize_rows(h)) @ wd.T)   # own scale per expert
        return ys
    layer._nvfp4_expert_outputs = f


def _bf16_matrix(big_endian=False, transposed=False):
    def f(blob, which, hidden, inter):
        off = formats.bf16_layout(hidden, inter)
        rows, K = (inter, hidden) if which in ("wg", "wu") else (hidden, inter)
        raw = np.asarray(blob, dtype=np.uint8)[off[which]: off[which] + 2 * rows * K].reshape(rows * K, 2)
        hi, lo = (raw[:, 0], raw[:, 1]) if big_endian else (raw[:, 1], raw[:, 0])
        bits = lo.astype(np.uint32) | (hi.astype(np.uint32) << 8)
        v = (bits << np.uint32(16)).view(np.float32).astype(np.float64)
        return v.reshape(K, rows).T.copy() if transposed else v.reshape(rows, K)
    formats.bf16_matrix = f


def bf16_big_endian():
    _bf16_matrix(big_endian=True)


def bf16_matrix_transposed():
    _bf16_matrix(transposed=True)


# ---------------------------------------------------------------------------
# LRU
# ---------------------------------------------------------------------------

def _step(victim_mru=False, victim_may_be_in_step=False, slot_highest=False, hit_touches=True):
    def step(self, lay, experts):
        S = sorted(set(int(e) for e in experts))
        if len(S) > self.capacity:
            raise lru.NoSpace(f"{len(S)} experts > capacity {self.capacity}")
        in_S = {(lay, e) for e in S}
        ev = []
        for e in S:
            key = (lay, e)
            if key in self.slot:
                if hit_touches:
                    self.order.remove(key)
                    self.order.append(key)
                ev.append((lru.HIT, lay, e, self.slot[key], -1))
                continue
            if len(self.order) == self.capacity:
                cands = [k for k in self.order if victim_may_be_in_step or k not in in_S]
                victim = cands[-1] if victim_mru else cands[0]
                self.order.remove(victim)
                s = self.slot.pop(victim)
                ev.append((lru.EVICT, victim[0], victim[1], s, -1))
            else:
                free = self._free_slots()
                s = max(free) if slot_highest else min(free)
            self.slot[key] = s
            self.order.append(key)
            ev.append((lru.MISS, lay, e, s, -1))
        return ev
    lru.LRUCache.step = step


def _resize(evict_mru=False, move_descending=False, move_to_highest=False):
    def resize(self, capacity):
        capacity = int(capacity)
        if capacity < 0:
            raise lru.NoSpace("negative capacity")
        ev = []
        while len(self.order) > capacity:
            victim = self.order.pop(-1 if evict_mru else 0)
            s = self.slot.pop(victim)
            ev.append((lru.EVICT, victim[0], victim[1], s, -1))
        old = self.capacity
        self.capacity = capacity
        if capacity < old:
            movers = sorted(((s, k) for k, s in self.slot.items() if s >= capacity), reverse=move_descending)
            for s, k in movers:
                free = self._free_slots()
                dst = max(free) if move_to_highest else min(free)
                self.slot[k] = dst
                ev.append((lru.MOVE, k[0], k[1], dst, s))
        return ev
    lru.LRUCache.resize = resize


def lru_evicts_most_recent():
    _step(victim_mru=True)


def lru_may_evict_a_key_of_the_step():
    _step(victim_may_be_in_step=True)


def lru_takes_highest_free_slot():
    _step(slot_highest=True)


def lru_hit_does_not_touch():
    _step(hit_touches=False)


def lru_lookup_does_not_touch():
    def lookup(self, lay, expert):
        return self.slot.get((lay, int(expert)), -1)
    lru.LRUCache.lookup = lookup


def resize_evicts_most_recent():
    _resize(evict_mru=True)


def resize_moves_descending():
    _resize(move_descending=True)


def resize_moves_to_highest_free():
    _resize(move_to_highest=True)


MUTANTS = {f.__name__: f for f in (
    e2m1_magnitude, e2m1_negative_zero, ue8m0_bias, nibble_order, scale_atom_row_major, scale_word_byte_swapped,
    pack_high_nibble_first, dequant_rows_scales_tiled, bf16_decode_low_half,
    quant_emax_one, quant_ties_away, quant_sign_of_zero, bf16_ties_away, bf16_truncate, bf16_via_fp32,
    topk_ties_to_higher_id, topk_nan_on_top, weights_not_renormalised, weights_reversed, logits_lane_of_element,
    logits_fp32_partials, logits_left_to_right, permutation_unstable, offsets_inclusive,
    silu_sign, gate_up_swapped, mxfp4_x_not_quantised, mxfp4_h_not_quantised, shared_expert_dropped,
    e4m3_bias, e4m3_subnormal_as_normal, nvfp4_blocks_of_32, nvfp4_matrix_scale_dropped,
    nvfp4_matrix_scales_rotated, bf16_big_endian, bf16_matrix_transposed,
    nvfp4_act_blocks_of_32, nvfp4_act_tensor_scale_dropped, nvfp4_act_scale_ties_up, nvfp4_act_h_scale_per_expert,
    lru_evicts_most_recent, lru_may_evict_a_key_of_the_step, lru_takes_highest_free_slot, lru_hit_does_not_touch,
    lru_lookup_does_not_touch,
    resize_evicts_most_recent, resize_moves_descending, resize_moves_to_highest_free)}


def apply(name: str) -> None:
    if name not in MUTANTS:
        raise KeyError(f"unknown oracle mutant {name!r}")
    MUTANTS[name]()
