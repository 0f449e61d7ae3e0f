"""Pins of the fp64 oracle to things other than itself.

Each test checks an oracle function against hand-worked fixtures, brute
force on tiny inputs, closed forms, invariants or a library routine, chosen
so that a dropped term, a wrong sign or index, or a transposed operand fails
one of them.  CPU only.
"""
import itertools
import math
import os

import numpy as np
import pytest

import oracle as o
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_golden(name):
    meta, rows = {}, []
    for line in open(os.path.join(GOLDEN, name)):
        line = line.split("#")[0].strip()
        if not line:
            continue
        if ":" in line:
            key, val = line.split(":", 1)
            val = val.strip()
            if "*" in val:
                pat, n = val.split("*")
                val = pat.strip() * int(n)
            meta[key.strip()] = bytes.fromhex(val)
        else:
            rows.append([float(v) for v in line.split()])
    return meta, rows


# ------------------------------------------------------------ bit helpers ---
def test_bf16_fp16_decoding():
    assert o.bf16_to_f64(np.array([0x3F80, 0xC000, 0x4049, 0x0000]))\
        .tolist() == [1.0, -2.0, 3.140625, 0.0]
    bits = np.arange(0, 0x7C00, 7, dtype=np.uint16)      # finite fp16 values
    ref = bits.view(np.float16).astype(np.float64)        # numpy's decoder
    assert np.array_equal(o.fp16_to_f64(bits), ref)
    assert o.fp16_to_f64(np.array([0x00, 0x38], np.uint8))[0] == 0.5


def test_bf16_rounding_nearest_even():
    # 1 + 2^-8 is halfway between bf16 1.0 and 1+2^-7: ties to even (1.0).
    v = np.array([1.0 + 2**-8, 1.0 + 3 * 2**-8, -(1.0 + 2**-7), 1.0 + 2**-9])
    assert o.f64_to_bf16_bits(v).tolist() == [0x3F80, 0x3F82, 0xBF81, 0x3F80]


# --------------------------------------------------------- dequantisation ---
def test_sb3_hand_worked_superblock():
    meta, rows = _read_golden("sb3_superblock.txt")
    raw = np.frombuffer(meta["codes_hex"] + meta["scales_hex"] + meta["d_hex"],
                        np.uint8)
    assert raw.size == 102
    w = o.dequant_sb3(raw, 1, 256)[0]
    for i, exp in rows:
        assert w[int(i)] == exp, (i, w[int(i)], exp)


def _pack_bits(values, width):
    """Little-endian bit stream of unsigned fields (test-side encoder)."""
    acc = 0
    for i, v in enumerate(values):
        acc |= int(v) << (width * i)
    return acc.to_bytes((width * len(values) + 7) // 8, "little")


def test_sb3_every_subscale_and_code():
    # one super-block per (s, q) pair, all codes q and all sub-scales s,
    # d = 1: every weight must be (2s+1)(2q-7)/8.
    pairs = list(itertools.product(range(16), range(8)))
    codes = b"".join(_pack_bits([q] * 256, 3) for s, q in pairs)
    scales = b"".join(_pack_bits([s] * 8, 4) for s, q in pairs)
    d = np.full(len(pairs), 1.0, np.float16).tobytes()
    raw = np.frombuffer(codes + scales + d, np.uint8)
    w = o.dequant_sb3(raw, len(pairs), 256)
    for r, (s, q) in enumerate(pairs):
        assert np.all(w[r] == (2 * s + 1) * (2 * q - 7) / 8.0), (s, q)


def test_sb3_bit_positions_are_a_bijection():
    # Flipping code bit b of weight i (stream bit 3i+b) from the all-zero
    # codes changes weight i alone, by 2^(b+1) in units of d(2s+1)/8.
    rng = np.random.default_rng(1)
    s = rng.integers(0, 16, 8)
    scales = _pack_bits(s, 4)
    d = np.array([0.25], np.float16).tobytes()
    base = o.dequant_sb3(np.frombuffer(bytes(96) + scales + d, np.uint8),
                         1, 256)[0]
    seen = np.zeros((256, 3), int)
    for bit in range(768):
        codes = bytearray(96)
        codes[bit // 8] |= 1 << (bit % 8)
        w = o.dequant_sb3(np.frombuffer(bytes(codes) + scales + d, np.uint8),
                          1, 256)[0]
        diff = np.nonzero(w != base)[0]
        assert diff.size == 1
        i = int(diff[0])
        step = 0.25 * (2 * s[i // 32] + 1) / 8.0
        b = int(round(math.log2((w[i] - base[i]) / step))) - 1
        assert (w[i] - base[i]) == step * 2 ** (b + 1)
        seen[i, b] += 1
    assert np.all(seen == 1)
    assert np.all(seen.sum(1) == 3)


def test_sb2_hand_worked_superblock():
    meta, rows = _read_golden("sb2_superblock.txt")
    raw = np.frombuffer(meta["codes_hex"] + meta["scales_hex"] + meta["d_hex"],
                        np.uint8)
    assert raw.size == 70
    w = o.dequant_sb2(raw, 1, 256)[0]
    for i, exp in rows:
        assert w[int(i)] == exp, (i, w[int(i)], exp)


def test_sb2_every_subscale_and_code():
    # one super-block per (s, q), d = 1: every weight is (2s+1)(2q-3)/4
    pairs = list(itertools.product(range(16), range(4)))
    codes = b"".join(_pack_bits([q] * 256, 2) for s, q in pairs)
    scales = b"".join(_pack_bits([s] * 8, 4) for s, q in pairs)
    d = np.full(len(pairs), 1.0, np.float16).tobytes()
    w = o.dequant_sb2(np.frombuffer(codes + scales + d, np.uint8),
                      len(pairs), 256)
    for r, (s, q) in enumerate(pairs):
        assert np.all(w[r] == (2 * s + 1) * (2 * q - 3) / 4.0), (s, q)


def test_sb2_bit_positions_and_rows():
    # Code bit b of weight i is stream bit 2i+b: flipping it from the
    # all-zero codes raises weight i alone by 2^(b+1) units of d(2s+1)/4;
    # super-blocks follow one another along a row, then rows.
    rng = np.random.default_rng(4)
    s = rng.integers(0, 16, 8)
    scales = _pack_bits(s, 4)
    d = np.array([0.25], np.float16).tobytes()
    base = o.dequant_sb2(np.frombuffer(bytes(64) + scales + d, np.uint8),
                         1, 256)[0]
    assert np.all(base == -3 * 0.25 * (2 * np.repeat(s, 32) + 1) / 4.0)
    for bit in range(512):
        codes = bytearray(64)
        codes[bit // 8] |= 1 << (bit % 8)
        w = o.dequant_sb2(np.frombuffer(bytes(codes) + scales + d, np.uint8),
                          1, 256)[0]
        i, b = bit // 2, bit % 2
        assert np.nonzero(w != base)[0].tolist() == [i]
        assert w[i] - base[i] == 0.25 * (2 * s[i // 32] + 1) / 4.0 * 2 ** (b + 1)
    # 2 rows x 512 columns: super-block m = row * 2 + column // 256, its
    # codes, scale word and d in plane order
    q = rng.integers(0, 4, (4, 256))
    sc = rng.integers(0, 16, (4, 8))
    dd = np.array([0.5, 0.25, 1.0, 2.0], np.float16)
    raw = np.frombuffer(b"".join(_pack_bits(r, 2) for r in q) +
                        b"".join(_pack_bits(r, 4) for r in sc) +
                        dd.tobytes(), np.uint8)
    w = o.dequant_sb2(raw, 2, 512)
    for m in range(4):
        want = (dd[m].astype(np.float64) * (2 * np.repeat(sc[m], 32) + 1) *
                (2 * q[m] - 3) / 4.0)
        assert np.array_equal(w[m // 2, 256 * (m % 2):256 * (m % 2) + 256],
                              want)


def test_sb2_generated_planes_and_range():
    raw = synth.gen_tensor(0, 0, 0, "up", synth.SB2_256, 16, 512,
                           (0.002, 0.01))
    assert raw.size == 16 * 2 * 70
    w = o.dequant_sb2(raw, 16, 512)
    assert np.abs(w).max() <= 0.01 * 31 * 3 / 4 + 1e-12
    assert np.array_equal(w.astype(np.float32).astype(np.float64), w)
    # all four codes occur in the codes plane
    cb = raw[:16 * 2 * 64]
    assert {int(v) for k in range(4) for v in np.unique((cb >> 2 * k) & 3)} \
        == {0, 1, 2, 3}


def test_nl3_hand_worked_superblock():
    meta, rows = _read_golden("nl3_superblock.txt")
    raw = np.frombuffer(meta["codes_hex"] + meta["scales_hex"] +
                        meta["d_hex"] + meta["extra_hex"], np.uint8)
    assert raw.size == 103
    w = o.dequant_nl3(raw, 1, 256)[0]
    for i, exp in rows:
        assert w[int(i)] == exp, (i, w[int(i)], exp)


def test_nl3_every_subscale_code_and_shift():
    # one super-block per (s, q, e), d = 1: every weight is
    # (2s+1)(cb3[q]+e)/16 with the configured codebook written out here
    cb3 = [-15, -10, -6, -2, 1, 5, 9, 14]
    trip = list(itertools.product(range(16), range(8), range(2)))
    codes = b"".join(_pack_bits([q] * 256, 3) for s, q, e in trip)
    scales = b"".join(_pack_bits([s] * 8, 4) for s, q, e in trip)
    d = np.full(len(trip), 1.0, np.float16).tobytes()
    extra = bytes([0xFF if e else 0x00 for s, q, e in trip])
    raw = np.frombuffer(codes + scales + d + extra, np.uint8)
    w = o.dequant_nl3(raw, len(trip), 256)
    for r, (s, q, e) in enumerate(trip):
        assert np.all(w[r] == (2 * s + 1) * (cb3[q] + e) / 16.0), (s, q, e)


def test_nl3_shift_bits_and_code_positions():
    # Flipping shift bit j raises exactly the 32 weights of block j, by
    # d(2s_j+1)/16; flipping code bit b of weight i changes weight i alone.
    rng = np.random.default_rng(2)
    s = rng.integers(0, 16, 8)
    q = rng.integers(0, 8, 256)
    codes, scales = _pack_bits(q, 3), _pack_bits(s, 4)
    d = np.array([0.5], np.float16).tobytes()
    base = o.dequant_nl3(np.frombuffer(codes + scales + d + bytes(1),
                                       np.uint8), 1, 256)[0]
    for j in range(8):
        w = o.dequant_nl3(np.frombuffer(codes + scales + d + bytes([1 << j]),
                                        np.uint8), 1, 256)[0]
        diff = np.nonzero(w != base)[0]
        assert diff.tolist() == list(range(32 * j, 32 * j + 32))
        assert np.all(w[diff] - base[diff] == 0.5 * (2 * s[j] + 1) / 16.0)
    for bit in range(0, 768, 7):
        cb = bytearray(codes)
        cb[bit // 8] ^= 1 << (bit % 8)
        w = o.dequant_nl3(np.frombuffer(bytes(cb) + scales + d + bytes(1),
                                        np.uint8), 1, 256)[0]
        assert np.nonzero(w != base)[0].tolist() == [bit // 3]


def test_nl3_codebook_and_generated_range():
    assert o.NL3_CODEBOOK.tolist() == [-15, -10, -6, -2, 1, 5, 9, 14]
    raw = synth.gen_tensor(0, 0, 0, "up", synth.NL3_256, 16, 512,
                           (0.002, 0.01))
    assert raw.size == 16 * 2 * 103
    w = o.dequant_nl3(raw, 16, 512)
    assert np.abs(w).max() <= 0.01 * 31 * 15 / 16 + 1e-12
    # every weight exact in fp32 (|(2s+1)(cb3+e)| <= 465, d fp16)
    assert np.array_equal(w.astype(np.float32).astype(np.float64), w)
    # both shift values occur
    ex = raw[-32:]
    assert 0 < np.unpackbits(ex).sum() < 256


@pytest.mark.parametrize("fmt,col", [(o.NL4_B32, 1), (o.Q4_B32, 2)])
def test_b32_hand_worked_block(fmt, col):
    meta, rows = _read_golden("b32_block.txt")
    raw = np.frombuffer(meta["codes_hex"] + meta["d_hex"], np.uint8)
    w = o.dequant_b32(fmt, raw, 1, 32)[0]
    for r in rows:
        assert w[int(r[0])] == r[col]


def test_b32_layout_rows_and_blocks():
    # two rows x 64 columns: block b of row r has d = r*2 + b + 1 and every
    # nibble of the row equal to (r + 3); blocks must not mix.
    rows, cols = 2, 64
    codes = b"".join(bytes([(r + 3) | ((r + 3) << 4)]) * (cols // 2)
                     for r in range(rows))
    d = np.array([1, 2, 3, 4], np.float16).tobytes()
    raw = np.frombuffer(codes + d, np.uint8)
    w = o.dequant_b32(o.Q4_B32, raw, rows, cols)
    for r in range(rows):
        for b in range(2):
            assert np.all(w[r, 32 * b:32 * b + 32] == (2 * r + b + 1) * (r - 5))


def test_nl4_codebook_is_the_configured_one():
    assert o.NL4_CODEBOOK.tolist() == [-127, -104, -83, -65, -49, -35, -22,
                                       -10, 1, 13, 25, 38, 53, 69, 89, 113]


def test_generated_tensor_dequant_ranges():
    # generated SB3 weights: |w| <= d_max*31*7/8, and they are exact in fp32
    raw = synth.gen_tensor(0, 0, 0, "up", synth.SB3_256, 16, 512, (0.002, 0.01))
    w = o.dequant_sb3(raw, 16, 512)
    assert np.abs(w).max() <= 0.01 * 31 * 7 / 8 + 1e-12
    assert np.array_equal(w.astype(np.float32).astype(np.float64), w)
    raw = synth.gen_tensor(0, 0, 0, "down", synth.NL4_B32, 16, 64, (0.002, 0.01))
    w = o.dequant_b32(o.NL4_B32, raw, 16, 64)
    assert np.array_equal(w.astype(np.float32).astype(np.float64), w)


# ---------------------------------------------------------------- routing ---
def _brute_topk(scores, k):
    out = []
    for row in scores:
        left = list(range(len(row)))
        sel = []
        for _ in range(k):
            best = left[0]
            for e in left[1:]:
                if row[e] > row[best]:      # strict: ties keep the lower index
                    best = e
            sel.append(best)
            left.remove(best)
        out.append(sel)
    return np.array(out)


def test_topk_matches_brute_force_and_ties():
    rng = np.random.default_rng(0)
    s = rng.standard_normal((20, 33))
    s[3, [4, 9, 20]] = 5.0              # three-way tie at the top
    s[5] = 0.0                          # all equal: 0..k-1
    s[7, [2, 30]] = s[7].max() + 1      # tie at the top, far apart
    ids = o.topk_select(s, 6)
    assert np.array_equal(ids, _brute_topk(s, 6))
    assert ids[3, :3].tolist() == [4, 9, 20]
    assert ids[5].tolist() == [0, 1, 2, 3, 4, 5]
    assert ids[7, :2].tolist() == [2, 30]


def test_route_weights_closed_forms():
    rng = np.random.default_rng(1)
    l = rng.standard_normal((6, 16)) * 2
    idx, w = o.route(l, 4)
    assert np.allclose(w.sum(1), 1.0, atol=1e-15)
    assert np.all(np.diff(w, axis=1) <= 0)          # sorted by weight
    # k = 2: w0 = sigmoid(l_a - l_b)
    idx2, w2 = o.route(l, 2)
    a = np.take_along_axis(l, idx2.astype(int), 1)
    assert np.allclose(w2[:, 0], 1 / (1 + np.exp(-(a[:, 0] - a[:, 1]))),
                       rtol=1e-14)
    # k = E: the weights are the softmax itself (scipy as the library routine)
    from scipy.special import softmax as sp_softmax
    idxE, wE = o.route(l, 16)
    ref = np.take_along_axis(sp_softmax(l, axis=1), idxE.astype(int), 1)
    assert np.allclose(wE, ref, rtol=1e-13)
    # a bias that is constant across experts changes nothing
    x = rng.standard_normal((3, 8))
    wr = rng.standard_normal((16, 8))
    l1 = o.router_logits(x, wr, None)
    l2 = o.router_logits(x, wr, np.full(16, 3.5))
    assert np.array_equal(o.route(l1, 3)[0], o.route(l2, 3)[0])


def test_router_logits_brute_force():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((3, 5))
    wr = rng.standard_normal((4, 5))
    b = rng.standard_normal(4)
    l = o.router_logits(x, wr, b)
    for t in range(3):
        for e in range(4):
            ref = math.fsum(x[t, h] * wr[e, h] for h in range(5)) + b[e]
            assert abs(l[t, e] - ref) < 1e-13


def test_group_pairs_brute_force():
    rng = np.random.default_rng(3)
    T, k, E = 9, 3, 7
    idx = np.array([rng.choice(E, k, replace=False) for _ in range(T)])
    off, pairs, active = o.group_pairs(idx, E)
    exp_pairs, exp_off = [], [0]
    for e in range(E):
        for t in range(T):
            for j in range(k):
                if idx[t, j] == e:
                    exp_pairs.append(t * k + j)
        exp_off.append(len(exp_pairs))
    assert pairs.tolist() == exp_pairs
    assert off.tolist() == exp_off
    assert active.tolist() == [e for e in range(E) if exp_off[e + 1] > exp_off[e]]
    assert sorted(pairs.tolist()) == list(range(T * k))


# -------------------------------------------------------------------- FFN ---
def test_silu_identities():
    z = np.array([-30.0, -2.0, -0.5, 0.0, 0.5, 2.0, 30.0])
    s = o.silu(z)
    assert s[3] == 0.0
    assert np.allclose(s - o.silu(-z), z, rtol=1e-15, atol=1e-15)
    for zi, si in zip(z, s):
        assert abs(si - zi / (1 + math.exp(-zi))) <= 1e-15 * max(1, abs(zi))


def test_expert_ffn_brute_force():
    rng = np.random.default_rng(4)
    n, H, F = 2, 6, 4
    x = rng.standard_normal((n, H))
    wu, wg = rng.standard_normal((F, H)), rng.standard_normal((F, H))
    wd = rng.standard_normal((H, F))
    h, y = o.expert_ffn(x, wu, wg, wd)
    for t in range(n):
        hh = []
        for f in range(F):
            u = math.fsum(wu[f, i] * x[t, i] for i in range(H))
            g = math.fsum(wg[f, i] * x[t, i] for i in range(H))
            hh.append(g / (1 + math.exp(-g)) * u)
        assert np.allclose(h[t], hh, rtol=1e-13)
        for r in range(H):
            ref = math.fsum(wd[r, f] * hh[f] for f in range(F))
            assert abs(y[t, r] - ref) <= 1e-12 * (1 + abs(ref))


def test_combine_brute_force():
    rng = np.random.default_rng(5)
    T, k, H = 3, 2, 5
    y = rng.standard_normal((T * k, H))
    w = rng.random((T, k))
    res = rng.standard_normal((T, H))
    out = o.combine(y, w, res)
    for t in range(T):
        for h in range(H):
            ref = res[t, h] + sum(w[t, j] * y[t * k + j, h] for j in range(k))
            assert abs(out[t, h] - ref) < 1e-13


def test_rmsnorm_unit_rms():
    r = np.random.default_rng(6).standard_normal((4, 3072)) * 37
    x = o.rmsnorm(r)
    assert np.allclose(np.sqrt(np.mean(x * x, 1)), 1.0, rtol=1e-6)


def test_tiny_layer_against_loops():
    """The whole tiny layer against a loop-by-loop restatement."""
    shp = synth.TINY
    x = o.bf16_to_f64(synth.gen_x(0, 8, shp.H))
    wr = o.bf16_to_f64(synth.gen_router(0, 0, shp.E, shp.H))
    src = o.ExpertSource(shp.H, shp.F, shp.fmt_up_gate, shp.fmt_down,
                         lambda e: synth.gen_expert_blob(shp, 0, 0, e))
    res = o.moe_layer(x, wr, None, shp.k, src)
    for t in range(8):
        logits = [math.fsum(x[t, h] * wr[e, h] for h in range(shp.H))
                  for e in range(shp.E)]
        order = sorted(range(shp.E), key=lambda e: (-logits[e], e))[:shp.k]
        assert res["topk_idx"][t].tolist() == order
        m = max(logits)
        ex = [math.exp(logits[e] - m) for e in order]
        ws = [v / sum(ex) for v in ex]
        out = np.zeros(shp.H)
        for j, e in enumerate(order):
            wu, wg, wd = src.weights(e)
            u = wu @ x[t]
            g = wg @ x[t]
            h = g / (1 + np.exp(-g)) * u
            out += ws[j] * (wd @ h)
        assert np.allclose(res["out"][t], out, rtol=1e-12, atol=1e-12)


# ------------------------------------------------------------- slot cache ---
class _LoopLRU:
    """A second, dictionary-based statement of the slot replay."""

    def __init__(self, cap, initial):
        self.slots = {s: (e, 0) for s, e in enumerate(initial[:cap])}
        for s in range(len(initial), cap):
            self.slots[s] = (None, 0)

    def step(self, chosen, stamp):
        chosen = sorted(set(chosen))
        where = {e: s for s, (e, _) in self.slots.items() if e is not None}
        touched, slot_of, misses, victims = set(), {}, [], []
        for e in chosen:
            if e in where:
                slot_of[e] = where[e]
                touched.add(where[e])
        for e in chosen:
            if e in where:
                continue
            cands = [(st, s) for s, (_, st) in self.slots.items()
                     if s not in touched]
            st, s = min(cands)
            self.slots[s] = (e, st)
            touched.add(s)
            slot_of[e] = s
            misses.append(e)
            victims.append(s)
        for s in touched:
            self.slots[s] = (self.slots[s][0], stamp)
        return slot_of, misses, victims


def test_slot_cache_matches_loop_replay_and_invariants():
    rng = np.random.default_rng(7)
    E, cap = 40, 12
    init = list(rng.permutation(E)[:cap])
    a = o.SlotCache(E, cap, init)
    b = _LoopLRU(cap, init)
    for step in range(1, 200):
        p = synth.zipf_popularity(E)
        chosen = rng.choice(E, 6, replace=True, p=p[rng.permutation(E)])
        ra = a.resolve(chosen, step)
        rb = b.step(list(int(c) for c in chosen), step)
        assert ra == rb
        slot_of, misses, victims = ra
        uniq = set(int(c) for c in chosen)
        assert set(slot_of) == uniq
        assert len(set(slot_of.values())) == len(uniq)   # no slot shared
        # table and owner are inverse maps
        for e in range(E):
            if a.table[e] >= 0:
                assert a.owner[a.table[e]] == e
        assert (a.table >= 0).sum() == (a.owner >= 0).sum()
        assert all(a.stamp[s] == step for s in slot_of.values())


def test_slot_cache_capacity_error():
    c = o.SlotCache(10, 2, [0, 1])
    with pytest.raises(RuntimeError):
        c.resolve(np.array([5, 6, 7]), 1)


# -------------------------------------------------------------- generator ---
def test_splitmix64_reference_values():
    # SplitMix64 seeded with 0 (state advanced by the golden gamma before
    # each output) starts 0xe220a8397b1dcdaf, 0x6e789e6aa1b965f4, ...
    w = synth.stream_words(0, 0, 3)
    assert [int(v) for v in w] == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4,
                                   0x06C45D188009454F]


def test_generated_scales_in_range():
    raw = synth.gen_tensor(3, 1, 2, "up", synth.SB3_256, 8, 256, (0.002, 0.01))
    d = o.fp16_to_f64(raw[-16:])
    assert np.all((d >= 0.002 - 1e-5) & (d <= 0.01 + 1e-5))
