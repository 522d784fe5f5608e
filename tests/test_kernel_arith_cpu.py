"""Bit-level identities the decode and prefill kernels rely on, checked exhaustively
on the CPU with numpy (the kernels themselves are checked against the oracle by the
GPU parity tests):

* int4 -> bf16 without a conversion: a nibble n of a 4-bit two's-complement q, put in
  the low mantissa bits of 0x4300 (128.0) after xor 8, is the bf16 value 136 + q.
* NVFP4 staging: every product of an e2m1 value and an e4m3 block scale is exact in
  f16 and in bf16, so the staged bf16 weight carries no rounding.
* The bf16 hi/lo split of the fp32 h that the tensor-core down projection reads:
  hi + lo equals h within 2^-17 relative.
"""
import numpy as np

import synth


def _bf16_bits_to_f32(bits):
    return (np.asarray(bits, dtype=np.uint32) << 16).view(np.float32)


def _e2m1(code):
    sign = -1.0 if code & 8 else 1.0
    e, m = (code >> 1) & 3, code & 1
    return sign * (m * 0.5 if e == 0 else (1 + m / 2) * 2.0 ** (e - 1))


def _e4m3(code):
    sign = -1.0 if code & 0x80 else 1.0
    e, m = (code >> 3) & 15, code & 7
    return sign * (m / 8 * 2.0 ** -6 if e == 0 else (1 + m / 8) * 2.0 ** (e - 7))


def test_int4_nibble_xor_gives_bf16_136_plus_q():
    # a 32-bit word holds nibbles 0..7; (w >> 4n) & 0x000F000F puts nibbles n and n+4
    # in the low bits of the two 16-bit halves, xor 0x4308 per half makes 136 + q
    rng = np.random.default_rng(0)
    words = np.concatenate([rng.integers(0, 2 ** 32, 4096, dtype=np.uint64).astype(np.uint32),
                            np.array([0, 0xFFFFFFFF, 0x88888888, 0x77777777], dtype=np.uint32)])
    for n in range(4):
        pair = ((words >> np.uint32(4 * n)) & np.uint32(0x000F000F)) ^ np.uint32(0x43084308)
        lo = _bf16_bits_to_f32(pair & np.uint32(0xFFFF)).astype(np.float64)
        hi = _bf16_bits_to_f32(pair >> np.uint32(16)).astype(np.float64)
        for half, nib in ((lo, n), (hi, n + 4)):
            q = ((words >> np.uint32(4 * nib)) & np.uint32(0xF)).astype(np.int64)
            q = np.where(q >= 8, q - 16, q)
            assert np.array_equal(half, 136.0 + q)


def test_e2m1_times_e4m3_is_exact_in_f16_and_bf16():
    e2 = [_e2m1(c) for c in range(16)]
    e4 = [_e4m3(c) for c in range(256) if (c & 0x7F) != 0x7F]      # 0x7F / 0xFF are NaN
    prod = np.array([a * b for a in e2 for b in e4], dtype=np.float64)
    # f16: the kernel multiplies the two as an f16 pair
    assert np.array_equal(prod.astype(np.float16).astype(np.float64), prod)
    # bf16: the staged weight
    bits = synth.round_bf16(prod.astype(np.float32))
    assert np.array_equal(_bf16_bits_to_f32(bits).astype(np.float64), prod)
    # and both factors are exact in f16 (the hardware conversions lose nothing)
    assert np.array_equal(np.array(e4).astype(np.float16).astype(np.float64), np.array(e4))


def test_bf16_hi_lo_split_keeps_h_within_2_pow_minus_17():
    rng = np.random.default_rng(1)
    h = np.concatenate([rng.standard_normal(200000) * s for s in (1e-3, 1.0, 30.0)]).astype(np.float32)
    h = np.concatenate([h, np.float32([0.0, -0.0, 1.0, -1.0, 65504.0, 1e-30, 3.0e38])])
    hi_bits = synth.round_bf16(h)
    hi = _bf16_bits_to_f32(hi_bits)
    r = (h - hi).astype(np.float32)          # exact in fp32: h and hi share the exponent range
    lo = _bf16_bits_to_f32(synth.round_bf16(r))
    got = hi.astype(np.float64) + lo.astype(np.float64)
    err = np.abs(got - h.astype(np.float64))
    assert np.all(err <= 2.0 ** -17 * np.abs(h.astype(np.float64)))
    # hi alone is the plain bf16 rounding (8 significant bits, 2^-8 relative): the split
    # adds the next 9 bits, since |h - hi| is at most half an ulp of hi
    assert np.all(np.abs(hi.astype(np.float64) - h) <= 2.0 ** -8 * np.abs(h.astype(np.float64)))
    assert np.max(err / np.maximum(np.abs(h.astype(np.float64)), 1e-300)) > 2.0 ** -19   # the bound is nearly reached


def test_nvfp4_expansion_writes_each_swizzled_chunk_once():
    # The NVFP4 prefill GEMM expands one stage (a B tile of 256 rows x 64 K elements) with
    # 128 threads, item = thread + 128 i (i < 4), row rr = item >> 1, half hf = item & 1:
    # it reads 16 code bytes at rr*32 + hf*16 of the raw tile and two scale bytes at
    # rr*16 + (kb & 3)*4 + 2*hf of the scale block, and writes chunk c = 4*hf + j (j < 4)
    # of row rr at rr*128 + ((c ^ (rr & 7)) * 16): the 128-byte swizzle the MMA descriptor
    # reads (TMA writes bf16 tiles the same way).  Every chunk of the 32 KB tile must be
    # written exactly once, at the address the swizzle gives K elements 8c .. 8c+7, and
    # every read must stay inside the 8 KB code tile and the 4 KB scale block.
    written = {}
    raw_reads, scale_reads = set(), set()
    for thread in range(128):
        for i in range(4):
            item = thread + 128 * i
            rr, hf = item >> 1, item & 1
            raw_reads.add(rr * 32 + hf * 16)
            for kb in range(4):
                off = rr * 16 + (kb & 3) * 4 + 2 * hf
                assert 0 <= off and off + 2 <= 256 * 16
                scale_reads.add(off)
            for j in range(4):
                c = 4 * hf + j
                addr = rr * 128 + ((c ^ (rr & 7)) * 16)
                assert addr not in written
                written[addr] = (rr, c)
    assert sorted(written) == list(range(0, 256 * 128, 16))
    for addr, (rr, c) in written.items():
        # the swizzle places chunk c of row rr at 16-byte position c ^ (rr % 8) of the row
        assert addr // 128 == rr and (addr % 128) // 16 == c ^ (rr % 8)
    assert sorted(raw_reads) == list(range(0, 256 * 32, 16))      # each 16-byte code group once
    assert len(scale_reads) == 256 * 2 * 4                        # two scales per item, per stage


def test_nvfp4_expansion_element_order():
    # Code byte b of a half-row holds K elements 2b (low nibble) and 2b+1 (high nibble); word j
    # (bytes 4j .. 4j+3) becomes output chunk j, whose 16-byte bf16 words are the pairs of bytes
    # 4j, 4j+1, 4j+2, 4j+3 in order: so chunk c of the row holds K elements 8c .. 8c+7 and the
    # 16-element block scale of elements 16s .. 16s+15 is block s (j < 2: s = 2 hf, else 2 hf + 1).
    for hf in range(2):
        for j in range(4):
            c = 4 * hf + j
            elems = [2 * (4 * j + b) + n for b in range(4) for n in range(2)]   # within the half
            assert [32 * hf + e for e in elems] == list(range(8 * c, 8 * c + 8))
            block = 2 * hf + (0 if j < 2 else 1)
            assert all((32 * hf + e) // 16 == block for e in elems)


def test_int4_nibbles_as_signed_bytes_16q():
    # The int8 tensor-core GEMV: (w << 4) & 0xF0F0F0F0 puts the even nibbles, w & 0xF0F0F0F0 the
    # odd ones, in the high halves of four bytes; read as signed int8 each byte is 16 q for the
    # two's-complement nibble q of its element (element 2i: low nibble of byte i).
    rng = np.random.default_rng(3)
    words = np.concatenate([rng.integers(0, 2 ** 32, 8192, dtype=np.uint64).astype(np.uint32),
                            np.array([0, 0xFFFFFFFF, 0x88888888, 0x77777777, 0x80808080], dtype=np.uint32)])
    even = ((words.astype(np.uint64) << 4) & 0xF0F0F0F0).astype(np.uint32)
    odd = words & np.uint32(0xF0F0F0F0)
    nib = np.stack([(words >> np.uint32(4 * e)) & np.uint32(15) for e in range(8)], axis=1).astype(np.int64)
    q = np.where(nib >= 8, nib - 16, nib)                       # element e of the word
    ev_bytes = even.view(np.int8).reshape(-1, 4).astype(np.int64)   # little-endian: byte i
    od_bytes = odd.view(np.int8).reshape(-1, 4).astype(np.int64)
    assert np.array_equal(ev_bytes, 16 * q[:, 0::2])
    assert np.array_equal(od_bytes, 16 * q[:, 1::2])


def _slice_rows(v):
    # the prep kernels' rule: E = exponent of max |v|, X = rint(v * 2^(14 - E)) clamped to
    # +-32767, hi = X >> 8 (signed), lo = X & 255, f = 2^(E - 14) / 16
    m = np.max(np.abs(v))
    E = int(np.frexp(np.float32(m))[1]) - 1 if m > 0 else 0
    X = np.clip(np.rint(v.astype(np.float64) * 2.0 ** (14 - E)), -32767, 32767).astype(np.int64)
    return X, X >> 8, X & 255, E


def test_int4_input_slices_block_fixed_point():
    rng = np.random.default_rng(4)
    for trial in range(20):
        scale = 10.0 ** rng.uniform(-6, 6)
        v = synth.round_bf16((rng.standard_normal(7168) * scale).astype(np.float32))
        v = _bf16_bits_to_f32(v).astype(np.float64)
        v[rng.integers(0, 7168, 5)] *= 0.0                          # exact zeros too
        X, hi, lo, E = _slice_rows(v)
        assert np.all(hi >= -128) and np.all(hi <= 127) and np.all(lo >= 0) and np.all(lo <= 255)
        assert np.array_equal(256 * hi + lo, X)                     # the two bytes rebuild X
        back = X * 2.0 ** (E - 14)
        big = np.abs(v) >= 2.0 ** (E - 7)                           # within 2^7 of the largest
        assert np.array_equal(back[big], v[big])                    # bf16 inputs there are exact
        assert np.max(np.abs(back - v)) <= 2.0 ** (E - 15)          # any input: half a step
    # fp32 inputs (h): the error of every element is at most half a step of 2^(E - 14)
    h = rng.standard_normal(2048) * 3.7
    X, hi, lo, E = _slice_rows(h)
    assert np.max(np.abs(X * 2.0 ** (E - 14) - h)) <= 2.0 ** (E - 15)


def test_int4_int8_mma_accumulators_fit_int32():
    # one 128-element group: 4 MMAs of 32 products each into int32; the largest |16 q| is 128,
    # the largest |hi| 128 and lo 255, so |256 D_hi + D_lo| < 2^31, and float(S) keeps 24 bits
    d_hi = 128 * 128 * 128
    d_lo = 128 * 128 * 255
    assert 256 * d_hi + d_lo < 2 ** 31


def test_int4_slice_permutation_matches_the_fragment_order():
    # MMA j of a group takes, per lane t, A = even16q / odd16q of word j (elements 32t + 8j +
    # {0,2,4,6} and +{1,3,5,7}); the sliced input stores every block of 8 elements even-first,
    # so bytes 0-3 of block j are elements {0,2,4,6} and bytes 4-7 are {1,3,5,7}
    def pos(e):
        return e >> 1 if e % 2 == 0 else 4 + (e >> 1)
    order = [None] * 8
    for e in range(8):
        order[pos(e)] = e
    assert order == [0, 2, 4, 6, 1, 3, 5, 7]


# ------------------------------------------------ NVFP4 decode on the f16 tensor cores --

def _mma_m16n8k16(a_regs, b_regs):
    """One mma.sync.m16n8k16 from per-lane fragments, as the PTX fragment layout defines
    them: a_regs[lane] = 4 pairs (a0..a3), b_regs[lane] = 2 pairs (b0, b1); returns D (16 x 8)."""
    A = np.zeros((16, 16))
    B = np.zeros((16, 8))
    for lane in range(32):
        g, t = lane >> 2, lane & 3
        a0, a1, a2, a3 = a_regs[lane]
        A[g, 2 * t:2 * t + 2] = a0
        A[g + 8, 2 * t:2 * t + 2] = a1
        A[g, 2 * t + 8:2 * t + 10] = a2
        A[g + 8, 2 * t + 8:2 * t + 10] = a3
        b0, b1 = b_regs[lane]
        B[2 * t:2 * t + 2, g] = b0
        B[2 * t + 8:2 * t + 10, g] = b1
    return A @ B


def test_nvfp4_mma_fragments_give_the_group_dot_products():
    # One 128-element group of 16 weight rows and 8 token columns through the kernel's
    # assignment: lane (g, t) holds code bytes 16t .. 16t+15 of rows g and g+8 (elements
    # 32t .. 32t+31); MMA j takes bytes 2j (a0 / a1) and 2j+1 (a2 / a3) times block scale
    # 2t + j // 4, and input elements 32t + 4j .. +3 of column g (b0, b1).  The 8 MMAs must
    # sum to the plain dot products.
    rng = np.random.default_rng(7)
    e2 = np.array([_e2m1(c) for c in range(16)])
    codes = rng.integers(0, 16, (16, 128))
    scodes = rng.integers(0, 0x7F, (16, 8))                    # e4m3, no NaN
    sv = np.array([[_e4m3(c) for c in row] for row in scodes])
    w = e2[codes] * np.repeat(sv, 16, axis=1)                 # value of each weight
    x = rng.standard_normal((128, 8)).astype(np.float16).astype(np.float64)
    D = np.zeros((16, 8))
    for j in range(8):
        a_regs, b_regs = [], []
        for lane in range(32):
            g, t = lane >> 2, lane & 3
            def pair(r, byte):
                e0 = 32 * t + 2 * byte                         # low nibble: the even element
                s = sv[r, 2 * t + j // 4]
                return np.array([e2[codes[r, e0]] * s, e2[codes[r, e0 + 1]] * s])
            a_regs.append((pair(g, 2 * j), pair(g + 8, 2 * j), pair(g, 2 * j + 1), pair(g + 8, 2 * j + 1)))
            k0 = 32 * t + 4 * j
            b_regs.append((x[k0:k0 + 2, g], x[k0 + 2:k0 + 4, g]))
        D += _mma_m16n8k16(a_regs, b_regs)
    assert np.allclose(D, w @ x, rtol=1e-12, atol=1e-12)


def test_nvfp4_input_slots_distinct_and_bank_conflict_free():
    # piece u (16 bytes) of lane (g, t) sits at slot (4u + t) ^ (4 (g & 1)) of column g's 256
    # bytes: one slot per piece, and the 8 lanes of a quarter-warp reading piece u hit 8
    # different 16-byte bank groups (a column's 256 bytes wrap the 128 bytes of banks twice)
    for g in range(8):
        slots = sorted((4 * u + t) ^ (4 * (g & 1)) for u in range(4) for t in range(4))
        assert slots == list(range(16))
    for u in range(4):
        for g0 in range(0, 8, 2):
            groups = {((g * 256 + 16 * ((4 * u + t) ^ (4 * (g & 1)))) % 128) // 16 for g in (g0, g0 + 1) for t in range(4)}
            assert len(groups) == 8


def test_nvfp4_inputs_as_f16_rows_with_a_power_of_two_scale():
    # x' = x * 2^(14 - E), E the exponent of the row's largest |x|: |x'| < 2^15 (f16 holds it);
    # a bf16 x is exact in f16 wherever |x| >= 2^(E - 28) (f16 normals); an fp32 h rounds to
    # 11 significant bits there (relative error at most 2^-11, half an ulp)
    rng = np.random.default_rng(8)
    for trial in range(20):
        scale = 10.0 ** rng.uniform(-8, 8)
        v = _bf16_bits_to_f32(synth.round_bf16((rng.standard_normal(4096) * scale).astype(np.float32)))
        v = v.astype(np.float64)
        m = np.max(np.abs(v))
        E = int(np.frexp(np.float32(m))[1]) - 1
        xs = v * 2.0 ** (14 - E)
        assert np.max(np.abs(xs)) < 2.0 ** 15
        f16 = xs.astype(np.float16).astype(np.float64)
        normal = np.abs(v) >= 2.0 ** (E - 28)
        assert np.array_equal(f16[normal], xs[normal])
        h = rng.standard_normal(2048) * scale
        E = int(np.frexp(np.float32(np.max(np.abs(h))))[1]) - 1
        hs = (h * 2.0 ** (14 - E)).astype(np.float32).astype(np.float64)
        hf = hs.astype(np.float16).astype(np.float64)
        big = np.abs(hs) >= 2.0 ** -14
        assert np.all(np.abs(hf[big] - hs[big]) <= 2.0 ** -11 * np.abs(hs[big]))


# ------------------------------------------------------- many-token router on tf32 MMAs --

def _tf32_rna(v):
    """fp32 -> tf32 (10 explicit mantissa bits), round to nearest, ties away from zero."""
    b = np.asarray(v, dtype=np.float32).view(np.uint32).astype(np.uint64)
    b = (b + 0x1000) & 0xFFFFE000
    return b.astype(np.uint32).view(np.float32)


def _tf32_trunc(v):
    """The bits the MMA reads of an fp32 operand: the top 10 explicit mantissa bits."""
    return (np.asarray(v, dtype=np.float32).view(np.uint32) & np.uint32(0xFFFFE000)).view(np.float32)


def test_router_tf32_split_is_within_2_pow_minus_21():
    # w = hi + lo with hi = tf32(w) and lo = w - hi (exact in fp32); the MMA reads lo's top
    # 11 significant bits, so hi + trunc(lo) is within 2^-21 |w|; a bf16 x is exact in tf32
    rng = np.random.default_rng(9)
    w = np.concatenate([rng.standard_normal(200000) * s for s in (1e-3, 0.02, 3.0)]).astype(np.float32)
    hi = _tf32_rna(w)
    lo = (w - hi).astype(np.float32)
    assert np.array_equal(hi.astype(np.float64) + lo.astype(np.float64), w.astype(np.float64))   # exact split
    got = hi.astype(np.float64) + _tf32_trunc(lo).astype(np.float64)
    assert np.all(np.abs(got - w) <= 2.0 ** -21 * np.abs(w.astype(np.float64)))
    x = _bf16_bits_to_f32(synth.round_bf16(rng.standard_normal(100000).astype(np.float32)))
    assert np.array_equal(_tf32_trunc(x), x)


def test_router_tf32_fragments_give_the_tile_logits():
    # one warp's 32 tokens x 32 experts over one k8 step, through the kernel's assignment
    # (a0 = x[g][t], a1 = x[g+8][t], a2 = x[g][t+4], a3 = x[g+8][t+4] of m-tile i; b0 = w[n][t],
    # b1 = w[n][t+4] with n = 8j + g; d_c -> token 16i + g + 8 (c >> 1), expert 8j + 2t + (c & 1))
    rng = np.random.default_rng(10)
    x = rng.standard_normal((32, 8))
    w = rng.standard_normal((32, 8))
    z = np.full((32, 32), np.nan)
    for i in range(2):
        for j in range(4):
            A = np.zeros((16, 8))
            B = np.zeros((8, 8))
            for lane in range(32):
                g, t = lane >> 2, lane & 3
                a = (x[16 * i + g, t], x[16 * i + g + 8, t], x[16 * i + g, t + 4], x[16 * i + g + 8, t + 4])
                A[g, t], A[g + 8, t], A[g, t + 4], A[g + 8, t + 4] = a          # the PTX A layout
                n = 8 * j + g
                B[t, g], B[t + 4, g] = w[n, t], w[n, t + 4]                      # the PTX B layout
            D = A @ B
            for lane in range(32):
                g, t = lane >> 2, lane & 3
                d = (D[g, 2 * t], D[g, 2 * t + 1], D[g + 8, 2 * t], D[g + 8, 2 * t + 1])   # the PTX D layout
                for c in range(4):
                    z[16 * i + g + 8 * (c >> 1), 8 * j + 2 * t + (c & 1)] = d[c]
    assert np.allclose(z, x @ w.T, rtol=1e-12, atol=1e-12)


def test_bf16_mma_fragments_give_the_group_dot_products():
    # The bf16 decode GEMV: lane (g, t) holds elements 8t .. 8t+7 of rows g and g+8 per group of
    # 32 (four words of two elements); MMA h takes words 2h (a0 / a1) and 2h+1 (a2 / a3), and B
    # words 2h, 2h+1 of the lane's 16 input bytes of column g (elements 8t + 4h .. +3).  The
    # two MMAs must sum to the plain dot products.
    rng = np.random.default_rng(11)
    w = rng.standard_normal((16, 32))
    x = rng.standard_normal((32, 8))
    D = np.zeros((16, 8))
    for h in range(2):
        a_regs, b_regs = [], []
        for lane in range(32):
            g, t = lane >> 2, lane & 3
            def word(row, wi):
                e0 = 8 * t + 2 * wi
                return w[row, e0:e0 + 2]
            a_regs.append((word(g, 2 * h), word(g + 8, 2 * h), word(g, 2 * h + 1), word(g + 8, 2 * h + 1)))
            k0 = 8 * t + 4 * h
            b_regs.append((x[k0:k0 + 2, g], x[k0 + 2:k0 + 4, g]))
        D += _mma_m16n8k16(a_regs, b_regs)
    assert np.allclose(D, w @ x, rtol=1e-12, atol=1e-12)
