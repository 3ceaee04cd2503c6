"""Pins of the CPU oracle against facts fixed outside the oracle itself:
closed forms, library routines (scipy's Hadamard, numpy's binary16), hand
worked examples under tests/golden/, invariants of the method, brute force on
tiny inputs, and the byte counts printed on the pages.  No GPU."""
import json
import math
import os

import numpy as np
import pytest
import scipy.linalg

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def fwht_loop(x):
    """Independent iterative butterfly transform, then the 1/sqrt(d) factor."""
    a = np.array(x, dtype=np.float64)
    h = 1
    while h < a.size:
        for i in range(0, a.size, 2 * h):
            for j in range(i, i + h):
                u, v = a[j], a[j + h]
                a[j], a[j + h] = u + v, u - v
        h *= 2
    return a / math.sqrt(a.size)


# ---------------------------------------------------------------- rotation

def test_hadamard_matches_scipy_and_is_orthogonal(orc):
    for d in (1, 2, 4, 16, 128):
        H = orc.hadamard(d).astype(np.int64)
        assert np.array_equal(H, scipy.linalg.hadamard(d))
        assert np.array_equal(H @ H.T, d * np.eye(d, dtype=np.int64))
        assert np.array_equal(H, H.T)


def test_rotation_closed_form_d4(orc):
    g = golden("hadamard4_example.json")
    assert np.array_equal(orc.rotate(np.array(g["x"], float)), np.array(g["Rx"], float))


def test_rotation_is_fwht_and_an_involution(orc):
    rng = np.random.default_rng(1)
    for _ in range(5):
        x = rng.standard_normal(128) * rng.choice([1.0, 30.0], 128)
        r = orc.rotate(x)
        assert np.allclose(r, fwht_loop(x), rtol=0, atol=1e-12)
        assert np.allclose(orc.rotate(r), x, rtol=0, atol=1e-12)
        assert math.isclose(np.dot(r, r), np.dot(x, x), rel_tol=1e-13)


def test_rotation_of_one_hot_is_flat(orc):
    x = np.zeros(128)
    x[0] = 3.0
    assert np.allclose(orc.rotate(x), 3.0 / math.sqrt(128), atol=1e-15)


# ---------------------------------------------------------------- binary16

def test_f16_from_double_matches_numpy(orc):
    rng = np.random.default_rng(2)
    vals = list(rng.standard_normal(3000) * 10.0 ** rng.uniform(-9, 5, 3000))
    # exact halfway points between adjacent binary16 values (ties to even)
    for bits in rng.integers(0, 0x7BFF, 400):
        a = float(np.uint16(bits).view(np.float16))
        b = float(np.uint16(bits + 1).view(np.float16))
        vals += [(a + b) / 2, -(a + b) / 2]
    vals += [0.0, -0.0, 65504.0, 65519.99, 65520.0, 1e6, -1e6, 2.0 ** -24, 2.0 ** -25, 2.0 ** -25 * 1.0001,
             2.0 ** -14, 2.0 ** -14 - 2.0 ** -25, 6.1e-5]
    for v in vals:
        want = int(np.array(v, dtype=np.float64).astype(np.float16).view(np.uint16))
        assert orc.f64_to_f16(v) == want, v


def test_f16_and_bf16_widening_match_numpy_and_torch(orc):
    import torch
    allbits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    f16 = allbits.view(np.float16).astype(np.float64)
    bf16 = torch.from_numpy(allbits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    for i in range(0, 65536, 7):
        if not np.isnan(f16[i]):
            assert orc.f16_to_f64(i) == f16[i]
        if not np.isnan(bf16[i]):
            assert orc.bf16_to_f64(i) == bf16[i]


# ---------------------------------------------------------------- quantiser

def test_worked_example_d4(orc):
    g = golden("quantize_d4_example.json")
    for normalize in (False, True):
        codes, S, Z, r = orc.quantize_vector(np.array(g["x"], float), g["bits"], normalize)
        assert np.array_equal(r, np.array(g["r"], float))
        assert orc.f16_to_f64(S) == g["S"] and orc.f16_to_f64(Z) == g["Z"]
        assert list(codes) == g["codes"]
        xh, rh = orc.dequantize_vector(codes, S, Z)
        assert np.array_equal(rh, np.array(g["rhat"], float))


def test_meta_exact_and_quotients_hand_values(orc):
    """The two checker helpers the parity rules rest on (the unrounded S, Z
    and the unrounded quotients) against values worked by hand."""
    g = golden("meta_quotients_d4.json")
    a = g["case_a"]
    assert np.array_equal(orc.rotate(np.array(a["x"], float)), np.array(a["r"], float))
    s_ex, z_ex = orc.meta_exact(np.array(a["x"], float), a["bits"], normalize=False)
    assert s_ex == a["s_exact"] and z_ex == a["z_exact"]
    s_ex, z_ex = orc.meta_exact(np.array(a["x"], float), a["bits"], normalize=True)
    assert math.isclose(s_ex, a["s_exact"], rel_tol=1e-14) and math.isclose(z_ex, a["z_exact"], rel_tol=1e-14)
    # 2 bits: the same range over 3 steps
    s2, z2 = orc.meta_exact(np.array(a["x"], float), 2, normalize=False)
    assert s2 == 4.0 / 3.0 and z2 == 1.0
    b = g["case_b"]
    assert orc.f16_to_f64(b["S_bits"]) == 0.5 and orc.f16_to_f64(b["Z_bits"]) == -1.0
    q = orc.quotients(np.array(b["r"], float), b["S_bits"], b["Z_bits"])
    assert np.array_equal(q, np.array(b["quotients"], float))
    # the codes of those quotients: ties to even (2.5 -> 2), clamped to 0..3
    assert list(orc.codes_given_meta(np.array(b["r"], float), 2, b["S_bits"], b["Z_bits"])) == [0, 2, 2, 3]


@pytest.mark.parametrize("bits", [4, 2, 8])
@pytest.mark.parametrize("normalize", [False, True])
def test_grid_exact_groups_are_recovered(orc, bits, normalize):
    rng = np.random.default_rng(10 + bits)
    top = (1 << bits) - 1
    for _ in range(40):
        S0 = float(np.float16(rng.uniform(0.01, 3.0)))
        Z0 = float(np.float16(rng.uniform(-20, 20)))
        c = rng.integers(0, top + 1, 128)
        c[rng.integers(128)] = 0
        c[rng.integers(128)] = top
        r = Z0 + S0 * c
        x = orc.rotate(r)  # R is its own inverse, so R x = r
        codes, S, Z, _ = orc.quantize_vector(x, bits, normalize)
        assert orc.f16_to_f64(S) == S0 and orc.f16_to_f64(Z) == Z0
        assert np.array_equal(codes, c)


def test_code_ranges_and_error_bound(orc, syn):
    x16 = syn.kv(5, syn.TID_K, 0, 64, 4, 128, 3, 10.0, 30.0, syn.F16)
    for bits in (4, 2, 8):
        top = (1 << bits) - 1
        for t in range(64):
            for h in range(4):
                x = x16[t, h].view(np.float16).astype(np.float64)
                codes, S, Z, r = orc.quantize_vector(x, bits)
                assert codes.min() == 0 and codes.max() == top
                s_ex, z_ex = orc.meta_exact(x, bits)
                s, z = orc.f16_to_f64(S), orc.f16_to_f64(Z)
                rh = s * codes + z
                bound = s / 2 + abs(z - z_ex) + top * abs(s - s_ex) + 1e-12
                assert np.max(np.abs(rh - r)) <= bound
                assert np.max(np.abs(rh - r)) <= 0.5 * s + abs(z - r.min()) + top * abs(s - s_ex) + 1e-12


def test_normalisation_on_off_invariant(orc, syn):
    """Per-vector standardisation cancels under g128 min/max RTN: codes and
    metadata agree with the un-normalised run except at ties / fp16 midpoints."""
    x16 = syn.kv(7, syn.TID_V, 0, 200, 2, 128, 3, 10.0, 30.0, syn.BF16)
    flips = 0
    total = 0
    for t in range(200):
        for h in range(2):
            x = (x16[t, h].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
            for bits in (4, 2, 8):
                c1, S1, Z1, r = orc.quantize_vector(x, bits, True)
                c0, S0, Z0, _ = orc.quantize_vector(x, bits, False)
                if (S1, Z1) != (S0, Z0):
                    s_ex, z_ex = orc.meta_exact(x, bits, True)
                    for v, a, b in ((s_ex, S1, S0), (z_ex, Z1, Z0)):
                        if a != b:
                            assert abs(int(a) - int(b)) == 1
                            ulp = abs(orc.f16_to_f64(a) - orc.f16_to_f64(b))
                            mid = (orc.f16_to_f64(a) + orc.f16_to_f64(b)) / 2
                            assert abs(v - mid) <= 1e-9 * ulp + 1e-300
                    continue
                q = orc.quotients(r, S1, Z1)
                diff = c1 != c0
                flips += int(diff.sum())
                total += 128
                if diff.any():
                    assert np.all(np.abs(np.abs(q[diff] - np.floor(q[diff])) - 0.5) < 1e-9)
    assert flips <= 1e-4 * total


def test_degenerate_groups(orc):
    codes, S, Z, _ = orc.quantize_vector(np.zeros(128), 4)
    assert S == 0 and Z == 0 and not codes.any()
    x = np.zeros(128)
    x[0] = 2.5  # R x is flat, so sigma = 0 is replaced by 1 and the range is 0
    codes, S, Z, _ = orc.quantize_vector(x, 2)
    assert S == 0 and not codes.any()
    assert orc.f16_to_f64(Z) == float(np.float16(2.5 / math.sqrt(128)))
    xh, _ = orc.dequantize_vector(codes, S, Z)
    assert np.allclose(xh, orc.rotate(np.full(128, orc.f16_to_f64(Z))), atol=0)


def test_codes_given_meta_clamps(orc):
    r = np.linspace(-1, 1, 128)
    S = orc.f64_to_f16(0.01)
    Z = orc.f64_to_f16(0.0)
    c = orc.codes_given_meta(r, 4, S, Z)
    assert c.min() == 0 and c.max() == 15
    assert np.all(c[r < 0] == 0) and np.all(c[r > 0.2] == 15)


# ---------------------------------------------------------------- layout

def test_segment_size_and_byte_layout(orc):
    g = orc.geom(num_blocks=3, num_kv_heads=2)
    assert orc.segment_bytes(g) == 1664
    assert orc.pool_bytes(g) == 3 * 2 * 1664
    pool = orc.new_pool(g, fill=0xFF)
    kc = np.arange(128) % 16
    vc = np.arange(128) % 4
    assert orc.pack_token(g, pool, 2, 5, 1, kc, 0x1234, 0x5678, vc, 0x9ABC, 0xDEF0) == 0
    seg = pool[(2 * 2 + 1) * 1664:(2 * 2 + 2) * 1664]
    # K row 5: element i at byte i/2, low nibble for even i
    assert list(seg[5 * 64:5 * 64 + 4]) == [0x10, 0x32, 0x54, 0x76]
    # V row 5: element i at byte i/4, bits 2*(i%4): codes 0,1,2,3 -> 0b11100100
    assert list(seg[1024 + 5 * 32:1024 + 5 * 32 + 2]) == [0xE4, 0xE4]
    # metadata arrays, little endian fp16 at offset 2*row
    assert list(seg[1536 + 10:1536 + 12]) == [0x34, 0x12]
    assert list(seg[1568 + 10:1568 + 12]) == [0x78, 0x56]
    assert list(seg[1600 + 10:1600 + 12]) == [0xBC, 0x9A]
    assert list(seg[1632 + 10:1632 + 12]) == [0xF0, 0xDE]
    # the neighbouring row and the other head are untouched
    assert np.all(seg[4 * 64:5 * 64] == 0xFF) and np.all(pool[:(2 * 2 + 1) * 1664] == 0xFF)
    back = orc.unpack_token(g, pool, 2, 5, 1)
    assert np.array_equal(back[0], kc) and np.array_equal(back[3], vc)
    assert back[1:3] == (0x1234, 0x5678) and back[4:] == (0x9ABC, 0xDEF0)
    assert orc.pack_token(g, pool, 3, 0, 0, kc, 0, 0, vc, 0, 0) == -5


@pytest.mark.parametrize("kb,vb", [(4, 4), (2, 2), (8, 4)])
def test_segment_layout_of_the_other_presets(orc, kb, vb):
    """Segment = 16 rows of kb-bit K codes, 16 rows of vb-bit V codes (element
    i of a b-bit row at bit b*i of the row, little-endian), then S_K, Z_K,
    S_V, Z_V as 16 fp16 each."""
    g = orc.geom(num_blocks=2, num_kv_heads=3, k_bits=kb, v_bits=vb)
    kr, vr = 128 * kb // 8, 128 * vb // 8
    seg_n = 16 * (kr + vr) + 4 * 32
    assert orc.segment_bytes(g) == seg_n and orc.pool_bytes(g) == 2 * 3 * seg_n
    pool = orc.new_pool(g, fill=0xFF)
    kc = (np.arange(128) * 7) % (1 << kb)
    vc = (np.arange(128) * 3) % (1 << vb)
    assert orc.pack_token(g, pool, 1, 9, 2, kc, 0x1111, 0x2222, vc, 0x3333, 0x4444) == 0
    seg = pool[(1 * 3 + 2) * seg_n:(1 * 3 + 3) * seg_n]

    def packed(codes, b):  # written out from the layout rule, one byte at a time
        out = []
        for byte in range(128 * b // 8):
            val = 0
            for i in range(128):
                bit0 = b * i
                for t in range(b):
                    if (bit0 + t) // 8 == byte and (codes[i] >> t) & 1:
                        val |= 1 << ((bit0 + t) % 8)
            out.append(val)
        return out

    assert list(seg[9 * kr:10 * kr]) == packed(kc, kb)
    assert list(seg[16 * kr + 9 * vr:16 * kr + 10 * vr]) == packed(vc, vb)
    meta = 16 * (kr + vr)
    for a, val in enumerate((0x1111, 0x2222, 0x3333, 0x4444)):
        assert list(seg[meta + 32 * a + 18:meta + 32 * a + 20]) == [val & 0xFF, val >> 8]
    assert np.all(seg[8 * kr:9 * kr] == 0xFF)
    back = orc.unpack_token(g, pool, 1, 9, 2)
    assert np.array_equal(back[0], kc) and np.array_equal(back[3], vc)
    assert back[1:3] == (0x1111, 0x2222) and back[4:] == (0x3333, 0x4444)


def test_append_skips_negative_slots_and_rejects_outside(orc, syn):
    g = orc.geom(num_blocks=2, num_kv_heads=1)
    pool = orc.new_pool(g, fill=0xAB)
    k = syn.kv(1, syn.TID_K, 0, 3, 1, 128, 0, 1, 1, syn.F16)
    v = syn.kv(1, syn.TID_V, 0, 3, 1, 128, 0, 1, 1, syn.F16)
    before = pool.copy()
    assert orc.quantize_append(g, pool, k, v, orc.F16, np.array([-1, -1, -1], np.int32)) == 0
    assert np.array_equal(pool, before)
    assert orc.quantize_append(g, pool, k, v, orc.F16, np.array([0, 32, 1], np.int32)) == -5


# ---------------------------------------------------------------- attention

def _build_pool(orc, syn, wl):
    g = orc.geom(num_blocks=wl.num_blocks, num_kv_heads=wl.hkv, block_size=wl.bs)
    pool = orc.new_pool(g)
    k = wl.kv_rows(syn.TID_K, 0, wl.total_tokens)
    v = wl.kv_rows(syn.TID_V, 0, wl.total_tokens)
    assert orc.quantize_append(g, pool, k, v, wl.dtype, wl.slots()) == 0
    return g, pool, k, v


def _to_f64(bits, dtype, syn):
    if dtype == syn.F16:
        return bits.view(np.float16).astype(np.float64)
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def test_attention_brute_force_tiny(orc, syn):
    """Explicit dequantisation with scipy's Hadamard and a hand softmax in
    numpy, against the oracle reading the paged, packed pool."""
    wl = syn.Workload("t", 2, 4, 2, 128, [37, 3], 16, syn.BF16, 3, 10.0, 30.0, seed=3)
    g, pool, k, v = _build_pool(orc, syn, wl)
    q = wl.query()
    out = orc.decode_attention(g, pool, q, wl.dtype, wl.block_table, wl.seq_lens)
    R = scipy.linalg.hadamard(128) / math.sqrt(128)
    for b in range(wl.batch):
        L = int(wl.seq_lens[b])
        for j in range(wl.hq):
            h = j // (wl.hq // wl.hkv)
            K = np.zeros((L, 128))
            V = np.zeros((L, 128))
            for t in range(L):
                row = wl.token_offsets[b] + t
                for M, src, bits in ((K, k, 4), (V, v, 2)):
                    x = _to_f64(src[row, h], wl.dtype, syn)
                    c, S, Z, _ = orc.quantize_vector(x, bits)
                    M[t] = R @ (orc.f16_to_f64(S) * c + orc.f16_to_f64(Z))
            s = K @ _to_f64(q[b, j], wl.dtype, syn) / math.sqrt(128)
            p = np.exp(s - s.max())
            want = (p / p.sum()) @ V
            assert np.allclose(out[b, j], want, rtol=0, atol=1e-12)


def test_window_rows_hand_example(orc):
    """A bf16 window of 2 sink and 3 recent rows ("Kompresja pamięci
    podręcznej KV..." (encorp.ai), OSCAR section), worked by hand: tokens 0..6
    of sequence 1 appended in order leave sink rows = tokens 0, 1 and ring rows
    (t % 3) = tokens 6, 4, 5; sequence 0 is untouched and a token with sequence
    id -1 is skipped."""
    d, hkv, sink, recent = 4, 1, 2, 3
    win = orc.new_window(2, hkv, sink, recent, d=d, fill=0xFFFF)
    k = np.array([[[10 * t + i for i in range(d)]] for t in range(8)], dtype=np.uint16)
    v = k + 1000
    orc.window_append(win, sink, recent, k, v, [1] * 7 + [-1], list(range(7)) + [3])
    rows = {0: 0, 1: 1, 2: 6, 3: 4, 4: 5}  # window row -> token, by hand
    for r, t in rows.items():
        assert list(win[1, 0, r, 0]) == [10 * t + i for i in range(d)]
        assert list(win[1, 0, r, 1]) == [1000 + 10 * t + i for i in range(d)]
    assert (win[0] == 0xFFFF).all()
    with pytest.raises(RuntimeError):
        orc.window_append(win, sink, recent, k[:1], v[:1], [2], [0])  # no sequence 2


def test_window_decode_brute_force(orc, syn):
    """Attention with sink and recent tokens raw and the rest dequantized,
    written out with scipy's Hadamard and a hand softmax in numpy; the raw rows
    come from the workload, not from the window buffer."""
    wl = syn.Workload("t", 2, 4, 2, 128, [37, 3], 16, syn.BF16, 3, 10.0, 30.0, seed=3)
    g, pool, k, v = _build_pool(orc, syn, wl)
    q = wl.query()
    R = scipy.linalg.hadamard(128) / math.sqrt(128)
    for sink, recent in ((2, 5), (0, 9), (4, 0), (0, 0)):
        win = orc.new_window(wl.batch, wl.hkv, sink, recent)
        for b in range(wl.batch):
            L = int(wl.seq_lens[b])
            rows = wl.token_offsets[b] + np.arange(L)
            orc.window_append(win, sink, recent, k[rows], v[rows], [b] * L, list(range(L)))
        out = orc.decode_attention_window(g, pool, win, sink, recent, q, wl.dtype, wl.block_table, wl.seq_lens)
        for b in range(wl.batch):
            L = int(wl.seq_lens[b])
            for j in range(wl.hq):
                h = j // (wl.hq // wl.hkv)
                K = np.zeros((L, 128))
                V = np.zeros((L, 128))
                for t in range(L):
                    row = wl.token_offsets[b] + t
                    raw = t < sink or t >= L - recent if recent else t < sink
                    for M, src, bits in ((K, k, 4), (V, v, 2)):
                        x = _to_f64(src[row, h], wl.dtype, syn)
                        if raw:
                            M[t] = x
                        else:
                            c, S, Z, _ = orc.quantize_vector(x, bits)
                            M[t] = R @ (orc.f16_to_f64(S) * c + orc.f16_to_f64(Z))
                s = K @ _to_f64(q[b, j], wl.dtype, syn) / math.sqrt(128)
                p = np.exp(s - s.max())
                want = (p / p.sum()) @ V
                assert np.allclose(out[b, j], want, rtol=0, atol=1e-12), (sink, recent, b, j)
        if sink == 0 and recent == 0:
            assert np.array_equal(out, orc.decode_attention(g, pool, q, wl.dtype, wl.block_table, wl.seq_lens))


def test_threaded_decode_is_the_single_threaded_one(orc, syn):
    """The oracle's std::thread split over (sequence, kv head) pairs changes
    nothing: every pair is computed by one thread in the same order."""
    wl = syn.Workload("t", 3, 8, 2, 128, [50, 17, 33], 16, syn.BF16, 3, 10.0, 30.0, seed=9)
    g, pool, _, _ = _build_pool(orc, syn, wl)
    q = wl.query()
    one = orc.decode_attention(g, pool, q, wl.dtype, wl.block_table, wl.seq_lens, nthreads=1)
    for nt in (2, 4, 16):
        assert np.array_equal(one, orc.decode_attention(g, pool, q, wl.dtype, wl.block_table, wl.seq_lens,
                                                        nthreads=nt))
    win = orc.new_window(wl.batch, wl.hkv, 3, 9)
    assert np.array_equal(orc.decode_attention_window(g, pool, win, 3, 9, q, wl.dtype, wl.block_table, wl.seq_lens),
                          orc.decode_attention_window(g, pool, win, 3, 9, q, wl.dtype, wl.block_table, wl.seq_lens,
                                                      nthreads=5))


def test_folded_form_equals_plain_form(orc, syn):
    wl = syn.Workload("t", 3, 16, 2, 128, [50, 17, 1], 16, syn.BF16, 3, 10.0, 30.0, seed=4, extra_blocks=2)
    g, pool, _, _ = _build_pool(orc, syn, wl)
    q = wl.query()
    plain = orc.decode_attention(g, pool, q, wl.dtype, wl.block_table, wl.seq_lens, form=0)
    folded = orc.decode_attention(g, pool, q, wl.dtype, wl.block_table, wl.seq_lens, form=1, nthreads=3)
    assert np.max(np.abs(plain - folded)) < 1e-10


def test_attention_special_cases(orc, syn):
    wl = syn.Workload("t", 1, 2, 1, 128, [20], 16, syn.F16, 4, 20.0, 20.0, seed=5, shuffle=False)
    g, pool, k, v = _build_pool(orc, syn, wl)
    bt = wl.block_table[0]
    q = wl.query()
    # L = 1: the output is the single dequantized value vector
    c, S, Z, _ = orc.quantize_vector(_to_f64(v[0, 0], wl.dtype, syn), 2)
    v0, _ = orc.dequantize_vector(c, S, Z)
    assert np.allclose(orc.decode_one(g, pool, q[0, 0], wl.dtype, 2, 0, bt, 1), v0, atol=1e-13)
    # q = 0: all scores equal, the output is the mean of the dequantized values
    vh = np.array([orc.dequantize_vector(*orc.quantize_vector(_to_f64(v[t, 0], wl.dtype, syn), 2)[0:3])[0]
                   for t in range(20)])
    zero_q = np.zeros(128, dtype=np.uint16)
    assert np.allclose(orc.decode_one(g, pool, zero_q, wl.dtype, 2, 1, bt, 20), vh.mean(0), atol=1e-12)
    # L = 0: zeros
    assert not orc.decode_one(g, pool, q[0, 0], wl.dtype, 2, 0, bt, 0).any()


def test_block_table_is_only_indirection(orc, syn):
    a = syn.Workload("t", 2, 8, 1, 128, [40, 33], 16, syn.BF16, 3, 10.0, 30.0, seed=6, shuffle=False)
    b = syn.Workload("t", 2, 8, 1, 128, [40, 33], 16, syn.BF16, 3, 10.0, 30.0, seed=6, shuffle=True)
    assert not np.array_equal(a.block_table, b.block_table)
    ga, pa, _, _ = _build_pool(orc, syn, a)
    gb, pb, _, _ = _build_pool(orc, syn, b)
    q = a.query()
    oa = orc.decode_attention(ga, pa, q, a.dtype, a.block_table, a.seq_lens)
    ob = orc.decode_attention(gb, pb, q, b.dtype, b.block_table, b.seq_lens)
    assert np.array_equal(oa, ob)


def test_dense_attention_against_numpy(orc, syn):
    k = syn.kv(8, syn.TID_K, 0, 9, 2, 128, 0, 1, 1, syn.F16)
    v = syn.kv(8, syn.TID_V, 0, 9, 2, 128, 0, 1, 1, syn.F16)
    q = syn.normal(8, syn.TID_Q, 128, syn.F16)
    out = orc.attention_dense(k, v, orc.F16, q, orc.F16, 4, 3)
    K = k[:, 1].view(np.float16).astype(np.float64)
    V = v[:, 1].view(np.float16).astype(np.float64)
    s = K @ q.view(np.float16).astype(np.float64) / math.sqrt(128)
    p = np.exp(s - s.max())
    assert np.allclose(out, (p / p.sum()) @ V, atol=1e-12)


# ---------------------------------------------------------------- byte accounting

def test_llama70b_kv_bytes_from_the_page(orc):
    g = golden("llama70b_kv_bytes.json")
    m = g["model"]
    per_token = orc.dense_bytes_per_token(m["layers"], m["num_kv_heads"], m["head_dim"], m["bytes_per_elem"])
    assert per_token == 327680
    assert round(per_token / 2 ** 20, 2) == g["per_token_mib_approx"]
    assert per_token * 131072 / 2 ** 30 == g["at_128k_gib_approx"]
    assert per_token * 2 ** 20 / 1e9 > g["at_1m_gb_min"]


def test_capacity_ratio_within_the_claim(orc):
    g = golden("capacity_claim.json")
    packed = orc.packed_bytes_per_token_head(128, 4, 2)
    assert packed == 104
    assert g["ratio_min"] <= 2 * 128 * 2 / packed <= g["ratio_max"]


def test_pool_comparison_catches_a_planted_code_error(orc, syn):
    """The full-size checker (tests/helpers.compare_pools) on two oracle-written
    pools: identical pools pass; a code moved by two steps in the oracle's
    copy (a planted mistake, not a near-tie) fails; a flipped S fails."""
    import helpers
    wl = syn.Workload("cmp", 2, 4, 2, 128, [40, 21], 16, syn.BF16, 3, 10.0, 30.0, seed=5)
    T = wl.total_tokens
    k = wl.kv_rows(syn.TID_K, 0, T)
    v = wl.kv_rows(syn.TID_V, 0, T)
    slots = wl.slots()
    g = orc.geom(num_blocks=wl.num_blocks, num_kv_heads=wl.hkv)
    a = orc.new_pool(g)
    helpers.oracle_append_threaded(g, a, k, v, wl.dtype, slots, nthreads=3)
    b = orc.new_pool(g)
    assert orc.quantize_append(g, b, k, v, wl.dtype, slots) == 0
    assert np.array_equal(a, b)
    rep = helpers.QuantReport()
    helpers.compare_pools(rep, a, b, wl.num_blocks, wl.hkv, k, v, wl.dtype, slots)
    assert rep.ok() and rep.vectors == 2 * T * wl.hkv and rep.code_mismatches == 0
    # plant: token 7, head 1, key element 10 moved by two codes
    p_, o_ = divmod(int(slots[7]), 16)
    kc, Sk, Zk, vc, Sv, Zv = orc.unpack_token(g, a, p_, o_, 1)
    kc = kc.copy()
    kc[10] = (int(kc[10]) + 2) % 16
    bad = a.copy()
    orc.pack_token(g, bad, p_, o_, 1, kc, Sk, Zk, vc, Sv, Zv)
    rep = helpers.QuantReport()
    helpers.compare_pools(rep, bad, b, wl.num_blocks, wl.hkv, k, v, wl.dtype, slots)
    assert not rep.ok()
    # plant: a scale off by 8 ulps
    bad = a.copy()
    kc, Sk, Zk, vc, Sv, Zv = orc.unpack_token(g, a, p_, o_, 0)
    orc.pack_token(g, bad, p_, o_, 0, kc, Sk + 8, Zk, vc, Sv, Zv)
    rep = helpers.QuantReport()
    helpers.compare_pools(rep, bad, b, wl.num_blocks, wl.hkv, k, v, wl.dtype, slots)
    assert not rep.ok()
