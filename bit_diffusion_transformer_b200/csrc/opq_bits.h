// opq_bits.h — register-level bit tricks shared by the OPQ kernels.
//
// Everything here is __host__ __device__ so that a host-side harness can check
// it exhaustively without a GPU; on the device PRMT is the hardware byte
// permute (inline PTX, generic mode with sign replication).
//
// Packed format ("OPQ INT4 Z-Image" model card, "Technical details / storage
// format": 8 magnitudes per uint32, 32 signs per uint32): element 8j+i of a row
// is nibble i of code word j; element 32j+i is bit i of sign word j.
#pragma once
#include <stdint.h>

#if defined(__CUDACC__)
#define OPQ_HD __host__ __device__ __forceinline__
#else
#define OPQ_HD static inline
#endif

namespace opqbits {

// PRMT, generic mode: output byte i = source byte (sel_i & 7) of {b:a}, or, when
// sel_i & 8, that byte's top bit replicated over 8 bits. Only sel[15:0] is used.
OPQ_HD uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
#if defined(__CUDA_ARCH__)
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
    return r;
#else
    uint64_t src = ((uint64_t)b << 32) | a;
    uint32_t r = 0;
    for (int i = 0; i < 4; ++i) {
        uint32_t s = (sel >> (4 * i)) & 0xFu;
        uint32_t byte = (uint32_t)(src >> (8 * (s & 7u))) & 0xFFu;
        if (s & 8u) byte = (byte & 0x80u) ? 0xFFu : 0x00u;
        r |= byte << (8 * i);
    }
    return r;
#endif
}

// ---------------------------------------------------------------------------
// Quantize: 15 per-row thresholds as bf16 bit patterns, T[1..15] non-decreasing,
// T[k] = smallest bf16 magnitude m with round-half-even(15 (m/max)^alpha) >= k.
// P[k] = T[k] * 0x00010001 (the threshold in both 16-bit halves).
//
// quant_pair: codes of the two bf16 weights in w2 (low half, high half) by a
// 4-level binary search done on both halves at once. For a 16-bit half holding
// 0x8000 | |w| and a threshold t <= 0x8000, the 32-bit subtraction never borrows
// across halves and bit 15 (bit 31) of the difference is |w| >= t. PRMT turns
// those bits into 0x0000FFFF / 0xFFFF0000 masks that select the next level's
// thresholds. Returns q_lo in bits 0..3 and q_hi in bits 16..19.
// ---------------------------------------------------------------------------
OPQ_HD uint32_t sel_mask(uint32_t m, uint32_t a, uint32_t b) { return (a & m) | (b & ~m); }

OPQ_HD uint32_t quant_pair(uint32_t w2, const uint32_t (&P)[16]) {
    const uint32_t M2 = w2 | 0x80008000u;
    const uint32_t k3 = prmt(M2 - P[8], 0, 0xBB99u);                 // q >= 8
    const uint32_t t2 = sel_mask(k3, P[12], P[4]);
    const uint32_t k2 = prmt(M2 - t2, 0, 0xBB99u);                   // q >= 4 + 8c3
    const uint32_t hi2 = sel_mask(k2, P[14], P[10]);
    const uint32_t lo2 = sel_mask(k2, P[6], P[2]);
    const uint32_t t1 = sel_mask(k3, hi2, lo2);
    const uint32_t k1 = prmt(M2 - t1, 0, 0xBB99u);                   // next level
    const uint32_t a0 = sel_mask(k1, P[3], P[1]);
    const uint32_t a1 = sel_mask(k1, P[7], P[5]);
    const uint32_t a2 = sel_mask(k1, P[11], P[9]);
    const uint32_t a3 = sel_mask(k1, P[15], P[13]);
    const uint32_t b0 = sel_mask(k2, a1, a0);
    const uint32_t b1 = sel_mask(k2, a3, a2);
    const uint32_t t0 = sel_mask(k3, b1, b0);
    const uint32_t k0 = prmt(M2 - t0, 0, 0xBB99u);
    return (k3 & 0x00080008u) | (k2 & 0x00040004u) | (k1 & 0x00020002u) | (k0 & 0x00010001u);
}

// Same codes with the four comparisons done as packed bf16 compares (set.ge.u32.bf16x2:
// 0xFFFF in each half where a >= b, exact for subnormals, false for NaN), which leaves the
// integer pipe only the threshold selects. Here P[k] holds T[k] in both halves with +inf
// (0x7F80) as the unreachable level instead of 0x8000; for finite non-negative halves it
// returns exactly quant_pair's codes.
OPQ_HD uint32_t bf16x2_ge_mask(uint32_t a, uint32_t b) {
#if defined(__CUDA_ARCH__)
    uint32_t r;
    asm("set.ge.u32.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
#else
    uint32_t r = 0;
    for (int h = 0; h < 2; ++h) {
        const uint32_t ua = ((a >> (16 * h)) & 0xFFFFu) << 16, ub = ((b >> (16 * h)) & 0xFFFFu) << 16;
        float fa, fb;
        __builtin_memcpy(&fa, &ua, 4);
        __builtin_memcpy(&fb, &ub, 4);
        if (fa >= fb) r |= 0xFFFFu << (16 * h);
    }
    return r;
#endif
}

// 0xFFFF in each half where the bf16 value is < 0 (so -0.0 and NaN give 0).
OPQ_HD uint32_t bf16x2_neg_mask(uint32_t a) {
#if defined(__CUDA_ARCH__)
    uint32_t r;
    asm("set.lt.u32.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(0u));
    return r;
#else
    uint32_t r = 0;
    for (int h = 0; h < 2; ++h) {
        const uint32_t ua = ((a >> (16 * h)) & 0xFFFFu) << 16;
        float fa;
        __builtin_memcpy(&fa, &ua, 4);
        if (fa < 0.0f) r |= 0xFFFFu << (16 * h);
    }
    return r;
#endif
}

OPQ_HD uint32_t quant_pair_f(uint32_t w2, const uint32_t (&P)[16]) {
    const uint32_t a = w2 & 0x7FFF7FFFu;
    const uint32_t k3 = bf16x2_ge_mask(a, P[8]);                      // q >= 8
    const uint32_t k2 = bf16x2_ge_mask(a, sel_mask(k3, P[12], P[4]));   // q >= 4 + 8c3
    const uint32_t t1 = sel_mask(k3, sel_mask(k2, P[14], P[10]), sel_mask(k2, P[6], P[2]));
    const uint32_t k1 = bf16x2_ge_mask(a, t1);
    const uint32_t b0 = sel_mask(k2, sel_mask(k1, P[7], P[5]), sel_mask(k1, P[3], P[1]));
    const uint32_t b1 = sel_mask(k2, sel_mask(k1, P[15], P[13]), sel_mask(k1, P[11], P[9]));
    const uint32_t k0 = bf16x2_ge_mask(a, sel_mask(k3, b1, b0));
    return (k3 & 0x00080008u) | (k2 & 0x00040004u) | (k1 & 0x00020002u) | (k0 & 0x00010001u);
}

// 8 weights (4 bf16 pairs, elements 0..7) -> one code word, element i in nibble i.
OPQ_HD uint32_t pack_codes(uint32_t q0, uint32_t q1, uint32_t q2, uint32_t q3) {
    // q_p holds element 2p in bits 0..3 and element 2p+1 in bits 16..19
    const uint32_t t0 = q0 | (q0 >> 12), t1 = q1 | (q1 >> 12);
    const uint32_t t2 = q2 | (q2 >> 12), t3 = q3 | (q3 >> 12);
    return prmt(prmt(t0, t1, 0x0040u), prmt(t2, t3, 0x0040u), 0x5410u);
}

// ---------------------------------------------------------------------------
// Coding by table. For non-negative bf16 values the bit pattern is monotone in
// the value, so with a row's nondecreasing thresholds T_1..T_15 (bf16 bits) the
// code q(a) = #{k : T_k <= a} of a magnitude a <= mx depends only on d = mx - a,
// and is 0 from d_z = mx - T_1 + 1 on. A row's table holds q(mx - e) for the
// entries e = 0 .. d_z, one byte each, with q in both nibbles (q * 17).
// ---------------------------------------------------------------------------
// One table word from the level boundaries. With B_k = bits(max) - T_k + 1 (0 when level k is
// out of reach), q(e) = #{k : B_k > e}. For word w (entries 4w .. 4w + 3) inside a stretch of
// entries (lo, hi] of the table: c_full = #{k : B_k > hi} levels hold for every entry of the
// stretch, and each boundary B inside the stretch (lo < B <= hi) adds 1 to the entries e < B
// of the word, i.e. to its first clamp(B - 4w, 0, 4) bytes. `inside` lists those boundaries.
OPQ_HD uint32_t table_word_from_bounds(uint32_t c_full, const int *inside, int n_inside, uint32_t w) {
    uint32_t word = c_full * 0x01010101u;
    for (int i = 0; i < n_inside; ++i) {
        int c = inside[i] - (int)(4u * w);
        c = c < 0 ? 0 : (c > 4 ? 4 : c);
        word += c == 0 ? 0u : (0x01010101u >> (8 * (4 - c)));
    }
    return word;
}

// Per-half maximum of two bf16 pairs (max.bf16x2): for non-negative finite halves it is the
// larger bit pattern, so it serves as a packed unsigned 16-bit max on magnitudes; a NaN half
// gives the canonical NaN 0x7FFF.
OPQ_HD uint32_t bf16x2_max(uint32_t a, uint32_t b) {
#if defined(__CUDA_ARCH__)
    uint32_t r;
    asm("max.NaN.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
#else
    uint32_t r = 0;
    for (int h = 0; h < 2; ++h) {
        const uint32_t ua = ((a >> (16 * h)) & 0xFFFFu) << 16, ub = ((b >> (16 * h)) & 0xFFFFu) << 16;
        float fa, fb;
        __builtin_memcpy(&fa, &ua, 4);
        __builtin_memcpy(&fb, &ub, 4);
        uint32_t m;
        if (fa != fa || fb != fb) m = 0x7FFFu;
        else m = (fa >= fb ? ua : ub) >> 16;
        r |= m << (16 * h);
    }
    return r;
#endif
}

// The code byte of a magnitude pair a (sign bits cleared; element 2p in the low nibble, 2p + 1
// in the high nibble) from a row table at byte offset `base` of tb whose entries hold q in both
// nibbles: the low half's entry gives the low nibble, the high half's the high nibble. The clamp is
// done on the magnitudes: d = mmb - max(a, lo2) stays within [base, base + d_z] per half
// (lo2 = bits(max) - d_z and mmb = bits(max) + base in both halves; the caller keeps
// bits(max) + base below 2^16 and a <= bits(max) per half, so no half borrows from the other);
// the index of the high half comes from a multiply-high so that it issues on the FMA pipe.
OPQ_HD uint32_t table_byte_clamped(const uint8_t *tb, uint32_t a, uint32_t lo2, uint32_t mmb) {
    const uint32_t d = mmb - bf16x2_max(a, lo2);
#if defined(__CUDA_ARCH__)
    uint32_t hi;
    asm("mul.hi.u32 %0, %1, 65536;" : "=r"(hi) : "r"(d));
#else
    const uint32_t hi = d >> 16;
#endif
    return ((uint32_t)tb[d & 0xFFFFu] & 0x0Fu) | ((uint32_t)tb[hi] & 0xF0u);
}

// Four code bytes (each in the low byte of its word) -> one code word, byte p = b_p.
OPQ_HD uint32_t codes_word(uint32_t b0, uint32_t b1, uint32_t b2, uint32_t b3) {
    return prmt(prmt(b0, b1, 0x0040u), prmt(b2, b3, 0x0040u), 0x5410u);
}

// Other bit widths: the two codes of a magnitude pair a from a row table whose entries hold q
// itself (one byte each); clamping and offsets as table_byte_clamped.
OPQ_HD void table_pair_bytes(const uint8_t *tb, uint32_t a, uint32_t lo2, uint32_t mmb, uint32_t &q0, uint32_t &q1) {
    const uint32_t d = mmb - bf16x2_max(a, lo2);
#if defined(__CUDA_ARCH__)
    uint32_t hi;
    asm("mul.hi.u32 %0, %1, 65536;" : "=r"(hi) : "r"(d));
#else
    const uint32_t hi = d >> 16;
#endif
    q0 = tb[d & 0xFFFFu];
    q1 = tb[hi];
}

// The 8 BITS-bit codes q[0..7] of one vector as the vector's 8 BITS-bit piece of the row's
// little-endian bit stream: element e at bits e BITS .. e BITS + BITS - 1 of (hi:lo).
template <int BITS>
OPQ_HD void pack_chunk(const uint32_t (&q)[8], uint32_t &lo, uint32_t &hi) {
    lo = 0u;
    hi = 0u;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        const int pos = e * BITS;
        if (pos + BITS <= 32) {
            lo |= q[e] << pos;
        } else if (pos >= 32) {
            hi |= q[e] << (pos - 32);
        } else {
            lo |= q[e] << pos;
            hi |= q[e] >> (32 - pos);
        }
    }
}

// Four consecutive vectors (32 elements) make BITS words of the stream. Lane i of a quad holds
// the piece of vector i (bits 8 BITS i .. 8 BITS (i + 1) - 1 of the quad's stream) and, from its
// neighbour, the piece of vector i + 1; it writes the words that start inside its own piece,
// at most two. quad_word gives the t-th of them (t = 0, 1): false if there is none, else its
// word index in the quad and its value.
template <int BITS>
OPQ_HD bool quad_word(uint32_t lo, uint32_t hi, uint32_t nlo, uint32_t nhi, uint32_t i, uint32_t t, uint32_t &w,
                      uint32_t &word) {
    const uint32_t piece = 8u * BITS;
    const uint32_t b0 = piece * i;
    w = (b0 + 31u) / 32u + t;
    if (32u * w >= b0 + piece) return false;   // starts in the next lane's piece (or past the quad)
    const uint32_t off = 32u * w - b0;         // 0 .. piece - 1
    const uint64_t c = ((uint64_t)hi << 32) | lo, cn = ((uint64_t)nhi << 32) | nlo;
    word = (uint32_t)((c >> off) | (cn << (piece - off)));
    return true;
}

// Sign bits (bf16 sign bit set) of 8 weights held as 4 bf16 pairs -> bits 0..7.
OPQ_HD uint32_t sign_byte(uint32_t w0, uint32_t w1, uint32_t w2, uint32_t w3) {
    // gather the high byte of every bf16 (its top bit is the sign), then move the
    // four top bits to bits 28..31 with one multiply (no carries: the products
    // of distinct bits land on distinct positions)
    const uint32_t a = prmt(w0, w1, 0x7531u) & 0x80808080u;   // elements 0..3
    const uint32_t b = prmt(w2, w3, 0x7531u) & 0x80808080u;   // elements 4..7
    return ((a * 0x00204081u) >> 28) | (((b * 0x00204081u) >> 28) << 4);
}

// ---------------------------------------------------------------------------
// Decode: one code word (8 nibbles) and its 8 sign bits -> 8 bf16 values
// sign * LUT[q], as 4 packed pairs (element 2p in the low half of out[p]).
// The 16-entry bf16 table travels as byte planes: L[j] holds the low bytes of
// entries 4j..4j+3, H[j] their high bytes (every H byte has its top bit clear:
// the table is non-negative).
// ---------------------------------------------------------------------------
struct DecodeTable {
    uint32_t L[4];
    uint32_t H[4];
};

OPQ_HD void decode8(uint32_t c, uint32_t sb, const DecodeTable &T, uint32_t out[4]) {
    const uint32_t s = c & 0x77777777u;        // low 3 bits of every nibble
    const uint32_t c4 = c << 4;
    // nibbles 0..3
    {
        const uint32_t m = prmt(c, c4, 0x9D8Cu);   // 0xFF in byte i iff bit 3 of nibble i
        const uint32_t l = sel_mask(m, prmt(T.L[2], T.L[3], s), prmt(T.L[0], T.L[1], s));
        const uint32_t sg = ((sb & 0xFu) * 0x10204080u) & 0x80808080u;   // sign i -> bit 8i+7
        const uint32_t h = sel_mask(m, prmt(T.H[2], T.H[3], s), prmt(T.H[0], T.H[1], s)) | sg;
        out[0] = prmt(l, h, 0x5140u);
        out[1] = prmt(l, h, 0x7362u);
    }
    // nibbles 4..7
    {
        const uint32_t sh = s >> 16;
        const uint32_t m = prmt(c, c4, 0xBFAEu);
        const uint32_t l = sel_mask(m, prmt(T.L[2], T.L[3], sh), prmt(T.L[0], T.L[1], sh));
        const uint32_t sg = (((sb >> 4) & 0xFu) * 0x10204080u) & 0x80808080u;
        const uint32_t h = sel_mask(m, prmt(T.H[2], T.H[3], sh), prmt(T.H[0], T.H[1], sh)) | sg;
        out[2] = prmt(l, h, 0x5140u);
        out[3] = prmt(l, h, 0x7362u);
    }
}

// ---------------------------------------------------------------------------
// Pair-table decode. A 64 KiB shared-memory table holds, for every code byte b
// (two nibbles = two consecutive weights), the bf16 pair
//     value(b) = LUT[b & 15] | LUT[b >> 4] << 16
// and, for every sign byte s (signs of 8 consecutive weights = 4 pairs), a
// spread word
//     spread(s) = sum_p  s[2p] << (15 - p)  |  s[2p+1] << (31 - p)
// so that (spread(s) << p) & 0x80008000 is the sign mask of pair p.
// Entry b occupies bytes [256 b, 256 b + 256): 32 copies of value(b) at
// 256 b + 4 lane, then 32 copies of spread(b) at 256 b + 128 + 4 lane; each lane
// reads its own copy, so the 32 lanes of a warp hit 32 different banks.
// The byte offset of a lookup is built by one PRMT from the code (or sign) word
// and a per-lane word holding 4 lane (or 128 + 4 lane) in its low byte.
// ---------------------------------------------------------------------------
constexpr uint32_t kPairTableBytes = 256u * 256u;

OPQ_HD uint32_t pair_value(uint32_t b, const uint16_t (&lut)[16]) {
    return (uint32_t)lut[b & 15u] | ((uint32_t)lut[(b >> 4) & 15u] << 16);
}

OPQ_HD uint32_t sign_spread(uint32_t s) {
    uint32_t x = 0;
    for (int p = 0; p < 4; ++p) {
        x |= ((s >> (2 * p)) & 1u) << (15 - p);
        x |= ((s >> (2 * p + 1)) & 1u) << (31 - p);
    }
    return x;
}

// Byte offset of code byte p of c (value part) for the lane whose low byte is in lw.
OPQ_HD uint32_t pair_offset(uint32_t c, uint32_t lw, uint32_t p) { return prmt(c, lw, 0x5504u | (p << 4)); }

// 8 weights: code word c, sign word sw (byte j holds their signs), values from
// the table via `load(offset)`. lw = 4 lane, lw2 = 128 + 4 lane.
template <class Load>
OPQ_HD void decode8_table(uint32_t c, uint32_t sw, uint32_t j, uint32_t lw, uint32_t lw2, Load load,
                          uint32_t out[4]) {
    const uint32_t x = load(prmt(sw, lw2, 0x5504u | (j << 4)));
    out[0] = load(pair_offset(c, lw, 0)) ^ (x & 0x80008000u);
    out[1] = load(pair_offset(c, lw, 1)) ^ ((x << 1) & 0x80008000u);
    out[2] = load(pair_offset(c, lw, 2)) ^ ((x << 2) & 0x80008000u);
    out[3] = load(pair_offset(c, lw, 3)) ^ ((x << 3) & 0x80008000u);
}

#if defined(__CUDACC__)
// Builds the pair table at shared-memory address `tab` with `nwarps` warps, this one warp `w` of
// them. Warp store i (of 128) covers entries 2i and 2i + 1: lane l writes copies 4 (l & 7) ..
// 4 (l & 7) + 3 of part (l >> 3) & 1 (0 value, 1 spread) of entry 2i + (l >> 4) in one 16-byte
// store, so a warp store fills 512 contiguous bytes (no bank conflicts) and the loop loads nothing.
// The magnitudes come by shuffles: for 4 bits, m0 = bf16 bits of LUT[lane & 15] and entry b is the
// pair value(b); for other widths, m0 = LUT[lane], m1 = LUT[32 + lane] (codes 0 .. 2^BITS - 1)
// and entry q < 2^BITS holds the magnitude of code q in both halves (0 above).
template <int BITS = 4>
__device__ __forceinline__ void build_pair_table(uint32_t tab, int w, int nwarps, int lane, uint32_t m0,
                                                 uint32_t m1 = 0u) {
    for (int i = w; i < 128; i += nwarps) {
        const uint32_t b = 2u * (uint32_t)i + ((uint32_t)lane >> 4);
        uint32_t v;
        if (BITS == 4) {
            const uint32_t lo = __shfl_sync(0xFFFFFFFFu, m0, (int)(b & 15u));
            const uint32_t hi = __shfl_sync(0xFFFFFFFFu, m0, (int)(b >> 4));
            v = lo | (hi << 16);
        } else {
            const uint32_t a0 = __shfl_sync(0xFFFFFFFFu, m0, (int)(b & 31u));
            const uint32_t a1 = __shfl_sync(0xFFFFFFFFu, m1, (int)(b & 31u));
            v = b < (1u << BITS) ? (b < 32u ? a0 : a1) * 0x00010001u : 0u;
        }
        if ((lane >> 3) & 1) v = sign_spread(b);
        asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(tab + 512u * (uint32_t)i + 16u * (uint32_t)lane),
                     "r"(v)
                     : "memory");
    }
}
#endif

}  // namespace opqbits
