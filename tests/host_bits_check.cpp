// Exhaustive host-side check of the kernels' register bit tricks (opq_bits.h)
// against naive per-element loops. Built and run by tests/test_host_bits.py.
#include <cstdio>
#include <cstdlib>
#include <cstdint>
#include <random>
#include <algorithm>
#include <vector>
#include <type_traits>
#include "opq_bits.h"

using namespace opqbits;

static int fails = 0;
#define CHECK(c, ...) do { if (!(c)) { if (fails < 20) { std::printf(__VA_ARGS__); std::printf("\n"); } ++fails; } } while (0)

int main() {
    std::mt19937_64 rng(12345);
    // --- prmt emulation: a few hand-checked cases of the PTX generic mode
    CHECK(prmt(0x33221100u, 0x77665544u, 0x3210u) == 0x33221100u, "prmt identity");
    CHECK(prmt(0x33221100u, 0x77665544u, 0x7654u) == 0x77665544u, "prmt upper");
    CHECK(prmt(0x00008000u, 0u, 0x9999u) == 0xFFFFFFFFu, "prmt sign replicate");
    CHECK(prmt(0x00007F00u, 0u, 0x9999u) == 0x00000000u, "prmt sign replicate 0");
    // --- quant_pair: thresholds sorted, <= 0x8000, ties and repeats included
    for (int trial = 0; trial < 400; ++trial) {
        uint32_t T[16] = {0};
        for (int k = 1; k <= 15; ++k) {
            uint32_t r = (uint32_t)(rng() % 0x8001u);
            if (trial % 7 == 0) r = (uint32_t)(rng() % 40u) + 0x3F00u;    // crowded thresholds
            if (trial % 11 == 0 && k > 10) r = 0x8000u;                    // unreachable levels
            T[k] = r;
        }
        std::sort(T + 1, T + 16);
        if (trial == 0) for (int k = 1; k <= 15; ++k) T[k] = 0x8000u;       // max == 0 row
        uint32_t P[16];
        for (int k = 0; k < 16; ++k) P[k] = T[k] * 0x00010001u;
        const int step = (trial < 8) ? 1 : 37;
        for (uint32_t m = 0; m < 0x8000u; m += step) {
            uint32_t m2 = (uint32_t)(rng() & 0x7FFFu);
            uint32_t s1 = (uint32_t)(rng() & 1u), s2 = (uint32_t)(rng() & 1u);
            uint32_t w2 = (m | (s1 << 15)) | ((m2 | (s2 << 15)) << 16);
            uint32_t q2 = quant_pair(w2, P);
            uint32_t want_lo = 0, want_hi = 0;
            for (int k = 1; k <= 15; ++k) { want_lo += (m >= T[k]); want_hi += (m2 >= T[k]); }
            CHECK((q2 & 0xFFFFu) == want_lo && (q2 >> 16) == want_hi,
                  "quant_pair trial %d m %x m2 %x got %x want %x %x", trial, m, m2, q2, want_lo, want_hi);
            // the packed-compare form: +inf stands for the unreachable level; finite halves only
            // (codes of non-finite weights are unspecified)
            if (m < 0x7F80u && m2 < 0x7F80u) {
                uint32_t PF[16];
                for (int k = 0; k < 16; ++k) PF[k] = (T[k] == 0x8000u ? 0x7F80u : T[k]) * 0x00010001u;
                const uint32_t qf = quant_pair_f(w2, PF);
                CHECK(qf == q2, "quant_pair_f trial %d m %x m2 %x got %x want %x", trial, m, m2, qf, q2);
            }
        }
    }
    // bf16x2_neg_mask: w < 0 per half (negative zero and NaN are not negative)
    for (uint32_t a = 0; a < 0x10000u; ++a) {
        const bool neg = (a & 0x8000u) && (a & 0x7FFFu) != 0u && (a & 0x7FFFu) <= 0x7F80u;
        const uint32_t r = opqbits::bf16x2_neg_mask(a | (a << 16));
        CHECK(r == (neg ? 0xFFFFFFFFu : 0u), "bf16x2_neg_mask %x -> %x", a, r);
    }
    // bf16x2_ge_mask host emulation against plain float compares, subnormals and zeros included
    for (uint32_t a = 0; a < 0x7F80u; a += 3)
        for (uint32_t b : {0x0000u, 0x0001u, 0x007Fu, 0x0080u, 0x3F80u, 0x7F7Fu, 0x7F80u}) {
            const uint32_t r = bf16x2_ge_mask(a | (b << 16), b | (a << 16));
            CHECK((r & 0xFFFFu) == (a >= b ? 0xFFFFu : 0u) && (r >> 16) == (b >= a ? 0xFFFFu : 0u),
                  "bf16x2_ge_mask %x %x -> %x", a, b, r);
        }
    // --- pack_codes / sign_byte
    for (int trial = 0; trial < 100000; ++trial) {
        uint32_t q[8], w[4], want_code = 0, want_sb = 0;
        for (int i = 0; i < 8; ++i) { q[i] = (uint32_t)(rng() & 15u); want_code |= q[i] << (4 * i); }
        for (int p = 0; p < 4; ++p) w[p] = (uint32_t)rng();
        for (int i = 0; i < 8; ++i) want_sb |= ((w[i / 2] >> (i % 2 ? 31 : 15)) & 1u) << i;
        uint32_t code = pack_codes(q[0] | q[1] << 16, q[2] | q[3] << 16, q[4] | q[5] << 16, q[6] | q[7] << 16);
        CHECK(code == want_code, "pack_codes %x %x", code, want_code);
        uint32_t sb = sign_byte(w[0], w[1], w[2], w[3]);
        CHECK(sb == want_sb, "sign_byte %x %x", sb, want_sb);
    }
    // --- decode8: random non-negative bf16 tables, every code word pattern class
    for (int trial = 0; trial < 200; ++trial) {
        uint16_t lut[16];
        for (int q = 0; q < 16; ++q) lut[q] = (uint16_t)(rng() & 0x7FFFu);
        if (trial == 0) lut[0] = 0;
        DecodeTable T;
        for (int j = 0; j < 4; ++j) {
            T.L[j] = 0; T.H[j] = 0;
            for (int b = 0; b < 4; ++b) {
                T.L[j] |= (uint32_t)(lut[4 * j + b] & 0xFFu) << (8 * b);
                T.H[j] |= (uint32_t)(lut[4 * j + b] >> 8) << (8 * b);
            }
        }
        for (int rep = 0; rep < 5000; ++rep) {
            uint32_t c = (uint32_t)rng(), sb = (uint32_t)(rng() & 0xFFu);
            uint32_t out[4];
            decode8(c, sb, T, out);
            for (int i = 0; i < 8; ++i) {
                uint32_t q = (c >> (4 * i)) & 15u;
                uint32_t want = lut[q] | (((sb >> i) & 1u) << 15);
                uint32_t got = (out[i / 2] >> (16 * (i % 2))) & 0xFFFFu;
                CHECK(got == want, "decode8 c %x sb %x i %d got %x want %x", c, sb, i, got, want);
            }
        }
    }
    // --- pair-table decode: build the 64 KiB table exactly as the kernels lay it out
    {
        std::vector<uint32_t> table(kPairTableBytes / 4);
        for (int trial = 0; trial < 50; ++trial) {
            uint16_t lut[16];
            for (int q = 0; q < 16; ++q) lut[q] = (uint16_t)(rng() & 0x7FFFu);
            if (trial == 0) lut[0] = 0;
            for (uint32_t b = 0; b < 256; ++b)
                for (uint32_t r = 0; r < 32; ++r) {
                    table[(b * 256 + 4 * r) / 4] = pair_value(b, lut);
                    table[(b * 256 + 128 + 4 * r) / 4] = sign_spread(b);
                }
            for (int rep = 0; rep < 20000; ++rep) {
                const uint32_t lane = (uint32_t)(rng() & 31u);
                const uint32_t lw = 4 * lane, lw2 = 128 + 4 * lane;
                uint32_t c = (uint32_t)rng(), sw = (uint32_t)rng(), j = (uint32_t)(rng() & 3u);
                uint32_t out[4];
                bool lane_ok = true;
                auto load = [&](uint32_t off) -> uint32_t {
                    if (off >= kPairTableBytes || (off & 3u) || ((off % 128u) / 4u) != lane) lane_ok = false;
                    return table[(off % kPairTableBytes) / 4];
                };
                decode8_table(c, sw, j, lw, lw2, load, out);
                CHECK(lane_ok, "table offset outside the lane's copy");
                const uint32_t sb = (sw >> (8 * j)) & 0xFFu;
                for (int i = 0; i < 8; ++i) {
                    uint32_t q = (c >> (4 * i)) & 15u;
                    uint32_t want = lut[q] | (((sb >> i) & 1u) << 15);
                    uint32_t got = (out[i / 2] >> (16 * (i % 2))) & 0xFFFFu;
                    CHECK(got == want, "decode8_table c %x sw %x j %u i %d got %x want %x", c, sw, j, i, got, want);
                }
            }
        }
    }
    // --- the quantize kernel's per-row code table: built word by word from the level boundaries
    // in stretches of 32 words (one per lane, as the kernel's ballots do), every entry against
    // q(b) = #{k : T_k <= b}; and the lookup of every magnitude up to the max at several table
    // offsets. Thresholds nondecreasing: spread, crowded, repeated, unreachable.
    {
        auto count_le = [](const uint16_t *T, int b) {
            uint32_t q = 0;
            for (int k = 1; k < 16; ++k) q += (int)T[k] <= b ? 1u : 0u;
            return q;
        };
        const uint32_t TAB = 4096;
        std::vector<uint32_t> tabw(16 * TAB / 4);
        for (int trial = 0; trial < 600; ++trial) {
            uint32_t mx = (uint32_t)(rng() % 0x7F81u);
            if (trial % 9 == 0) mx = 0x7F80u;            // +inf max
            if (trial % 13 == 0) mx = (uint32_t)(rng() % 64u);   // subnormal-range max
            uint16_t T[16] = {0};
            if (mx == 0u || trial % 17 == 0) {
                for (int k = 1; k < 16; ++k) T[k] = 0x7F80u;   // an all-zero row: no level reachable
            } else {
                // T_15 <= mx; spread below it over up to 16 binades, or crowded near it
                std::vector<uint32_t> v(15);
                const uint32_t span = (trial % 5 == 0) ? 40u : 2048u + (uint32_t)(rng() % 2048u);
                for (auto &x : v) x = mx > span ? mx - (uint32_t)(rng() % span) : 1u + (uint32_t)(rng() % mx);
                if (trial % 7 == 0) v[3] = v[4] = v[5];        // repeated thresholds
                std::sort(v.begin(), v.end());
                for (int k = 1; k < 16; ++k) T[k] = (uint16_t)std::max<uint32_t>(1u, v[k - 1]);
            }
            const uint32_t T1 = T[1];
            const uint32_t dz = T1 <= mx ? mx - T1 + 1u : 0u;
            if (dz >= TAB) continue;                           // such rows take the search
            const uint32_t words = (dz + 4u) >> 2;
            int B[16];
            for (int k = 1; k < 16; ++k) B[k] = (int)T[k] <= (int)mx ? (int)mx - (int)T[k] + 1 : 0;
            CHECK((uint32_t)B[1] == dz, "B_1 != dz trial %d", trial);
            for (uint32_t slot : {0u, 7u, 15u}) {
                const uint32_t base = slot * TAB;
                if (base + 0x7F80u >= 0x10000u) continue;      // the kernels keep max + base below 2^16
                std::fill(tabw.begin(), tabw.end(), 0xEEEEEEEEu);
                const uint8_t *tb = reinterpret_cast<const uint8_t *>(tabw.data());
                for (uint32_t i0 = 0; i0 < words; i0 += 32u) {
                    const int lo = (int)(4u * i0), hi = lo + 127;
                    uint32_t c_full = 0;
                    int inside[16], n_in = 0;
                    for (int k = 1; k < 16; ++k) {
                        if (B[k] > hi) ++c_full;
                        else if (B[k] > lo) inside[n_in++] = B[k];
                    }
                    for (uint32_t w = i0; w < std::min(i0 + 32u, words); ++w)
                        tabw[base / 4 + w] = table_word_from_bounds(c_full, inside, n_in, w) * 0x11u;
                }
                for (uint32_t e = 0; e < 4u * words; ++e)
                    CHECK(tb[base + e] == 17u * count_le(T, (int)mx - (int)e), "table trial %d base %u e %u got %u want %u",
                          trial, base, e, tb[base + e], 17u * count_le(T, (int)mx - (int)e));
                const uint32_t mmb = (mx + base) * 0x00010001u, lo2 = (mx - dz) * 0x00010001u;
                const uint32_t step = mx > 20000u ? 7u : 1u;
                for (uint32_t a = 0; a <= mx; a += step) {
                    const uint32_t a2 = (uint32_t)(rng() % (mx + 1u));
                    const uint32_t b = table_byte_clamped(tb, a | (a2 << 16), lo2, mmb);
                    CHECK(b == (count_le(T, (int)a) | (count_le(T, (int)a2) << 4)), "table_byte_clamped %x %x mx %x",
                          a, a2, mx);
                }
            }
        }
    }
    // bf16x2_max on non-negative finite halves: the larger bit pattern
    for (int t = 0; t < 200000; ++t) {
        const uint32_t a = (uint32_t)(rng() % 0x7F81u), b = (uint32_t)(rng() % 0x7F81u);
        const uint32_t c = (uint32_t)(rng() % 0x7F81u), d = (uint32_t)(rng() % 0x7F81u);
        const uint32_t r = bf16x2_max(a | (c << 16), b | (d << 16));
        CHECK(r == (std::max(a, b) | (std::max(c, d) << 16)), "bf16x2_max %x %x %x %x -> %x", a, b, c, d, r);
    }
    // codes_word: byte p of the word is the low byte of b_p
    for (int t = 0; t < 1000; ++t) {
        const uint32_t b[4] = {(uint32_t)rng(), (uint32_t)rng(), (uint32_t)rng(), (uint32_t)rng()};
        const uint32_t want = (b[0] & 0xFFu) | ((b[1] & 0xFFu) << 8) | ((b[2] & 0xFFu) << 16) | ((b[3] & 0xFFu) << 24);
        CHECK(codes_word(b[0], b[1], b[2], b[3]) == want, "codes_word %x %x %x %x", b[0], b[1], b[2], b[3]);
    }
    // other bit widths: 32 random codes of a quad as pieces (pack_chunk) and the quad's words
    // (quad_word over its four lanes) against the bit stream written one bit at a time
    auto check_stream = [&](auto bits_tag) {
        constexpr int B = decltype(bits_tag)::value;
        for (int t = 0; t < 2000; ++t) {
            uint32_t q[32];
            for (int e = 0; e < 32; ++e) q[e] = (uint32_t)(rng() & ((1u << B) - 1u));
            if (t == 0) for (int e = 0; e < 32; ++e) q[e] = (1u << B) - 1u;   // all ones
            uint32_t want[B] = {};
            for (int e = 0; e < 32; ++e)
                for (int b = 0; b < B; ++b)
                    if ((q[e] >> b) & 1u) want[(e * B + b) / 32] |= 1u << ((e * B + b) % 32);
            uint32_t lo[5], hi[5];
            for (int i = 0; i < 4; ++i) {
                uint32_t qq[8];
                for (int e = 0; e < 8; ++e) qq[e] = q[8 * i + e];
                pack_chunk<B>(qq, lo[i], hi[i]);
            }
            lo[4] = (uint32_t)rng();   // the next quad's lane 0: must not matter
            hi[4] = (uint32_t)rng();
            int seen[B] = {};
            for (uint32_t i = 0; i < 4; ++i)
                for (uint32_t tt = 0; tt < 2; ++tt) {
                    uint32_t w = 0, word = 0;
                    if (!quad_word<B>(lo[i], hi[i], lo[i + 1], hi[i + 1], i, tt, w, word)) continue;
                    CHECK(w < (uint32_t)B, "quad_word<%d> word index %u", B, w);
                    if (w >= (uint32_t)B) continue;
                    ++seen[w];
                    CHECK(word == want[w], "quad_word<%d> t %d lane %u word %u got %x want %x", B, t, i, w, word, want[w]);
                }
            for (int w = 0; w < B; ++w) CHECK(seen[w] == 1, "quad_word<%d> word %d written %d times", B, w, seen[w]);
        }
    };
    check_stream(std::integral_constant<int, 3>{});
    check_stream(std::integral_constant<int, 4>{});
    check_stream(std::integral_constant<int, 5>{});
    check_stream(std::integral_constant<int, 6>{});
    // table_pair_bytes: both codes of a magnitude pair from a table of plain q bytes
    {
        std::vector<uint8_t> tb(0x10000);
        for (auto &b : tb) b = (uint8_t)(rng() & 63u);
        for (int t = 0; t < 20000; ++t) {
            const uint32_t mx = 0x3000u + (uint32_t)(rng() % 0x4000u), dz = 1u + (uint32_t)(rng() % 1500u);
            const uint32_t base = 4096u * (uint32_t)(rng() % 8u);
            if (mx + base >= 0x10000u || dz > mx) continue;
            const uint32_t a0 = (uint32_t)(rng() % (mx + 1u)), a1 = (uint32_t)(rng() % (mx + 1u));
            uint32_t q0 = 0, q1 = 0;
            table_pair_bytes(tb.data(), a0 | (a1 << 16), (mx - dz) * 0x00010001u, (mx + base) * 0x00010001u, q0, q1);
            const uint32_t e0 = mx - std::max(a0, mx - dz), e1 = mx - std::max(a1, mx - dz);
            CHECK(q0 == tb[base + e0] && q1 == tb[base + e1], "table_pair_bytes %x %x mx %x dz %u", a0, a1, mx, dz);
        }
    }
    std::printf("%s fails=%d\n", fails ? "FAIL" : "OK", fails);
    return fails ? 1 : 0;
}
