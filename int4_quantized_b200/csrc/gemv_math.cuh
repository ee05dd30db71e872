// gemv_math.cuh -- the arithmetic of the quantized GEMV, shared by the single-call GEMV
// (gemv.cu) and the persistent decode-stack kernel (stack.cu).
//
// A weight tile is 128 rows x 128 bytes of the packed payload (128-byte swizzle, as a 2D
// TMA load writes it). A consumer warp owns 16 rows of it; lane (g, t) reads L bytes of
// rows g and g + 8 per segment. Codes become exact bf16 values (A fragments), the
// activations exact bf16 pieces (B fragments, hi + mid + lo = x), and warp-level
// mma.sync m16n8k16 (bf16 x bf16 -> fp32) forms the group sums, which the group's fp32
// scale multiplies into fp32 totals ("Huit bits, puis quatre", "Ranger des entiers dans
// des f32": the products of the codes and the activations, scaled per group).
#pragma once

#include "common.cuh"

namespace q4 {
namespace gm {

constexpr int kTileBytes = 128;                    // bytes of a weight row per stage
constexpr int kTileRows = 128;                     // weight rows per tile (8 warps x 16)
constexpr int kTileWords = kTileBytes * kTileRows;  // 16 KB of codes per stage

// ---- activation pieces ---------------------------------------------------------------
// x = hi + mid + lo exactly, each piece a bf16 value held in the high half of an fp32
// word (its low 16 bits are zero). hi and mid are truncations, so x - hi and r - mid are
// exact fp32 differences; lo keeps at most 8 significant bits. Only activations below
// 2^-110 in magnitude can lose bits of lo (an error below 2^-126).
Q4_DEVINL void split3(float v, uint32_t (&pc)[3]) {
    const uint32_t hi = __float_as_uint(v) & 0xffff0000u;
    const float r = v - __uint_as_float(hi);
    const uint32_t mid = __float_as_uint(r) & 0xffff0000u;
    const float lo = r - __uint_as_float(mid);
    pc[0] = hi;
    pc[1] = mid;
    pc[2] = __float_as_uint(lo) & 0xffff0000u;
}

// bf16 pair (a in the low half, b in the high half) from two pieces.
Q4_DEVINL uint32_t pack_pair(uint32_t a, uint32_t b) { return prmt(a, b, 0x7632u); }

// Index (uint2 units) of the B fragment of MMA i of a stage, n8 block nb, lane.
Q4_DEVINL int frag_idx(int i, int nb, int lane, int NB, int lw, bool paired) {
    return paired ? ((((i >> 1) * NB + nb) * lw + lane) << 1) + (i & 1) : (i * NB + nb) * lw + lane;
}

// The B fragments of 8 consecutive k (offset kk inside the stage, a multiple of 8) of
// virtual activation row vm of a 16-row chunk: column P * vm + p holds piece p, for the
// columns that exist (< 8 * NB, and < 4 * NB... when only 16 lanes are stored). v = 0
// writes zero columns (rows past M). The k-slots of an MMA map onto memory k as the
// lane's A words do (see unpack_a): int4, MMA 2j of word j: slots (2t, 2t+1, 2t+8, 2t+9)
// = k (0, 4, 1, 5) of the word, MMA 2j + 1: k (2, 6, 3, 7); int8, word j: k (0, 2, 1, 3).
template <int BITS, int L>
Q4_DEVINL void frag_unit(uint2 *stage, int kk, int vm, const float (&v)[8], int P, int ncols, int NB, int lw,
                         bool paired) {
    constexpr int KTI = BITS == 4 ? L / 2 : L / 4;  // MMAs per segment
    uint32_t pc[3][8];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        uint32_t t3[3];
        split3(v[q], t3);
        pc[0][q] = P == 1 ? __float_as_uint(v[q]) & 0xffff0000u : t3[0];
        pc[1][q] = t3[1];
        pc[2][q] = t3[2];
    }
#pragma unroll
    for (int p = 0; p < 3; ++p) {
        if (p >= P) break;
        const int col = P * vm + p;
        if (col >= ncols) break;
        const int nb = col >> 3, lb = 4 * (col & 7);
        if constexpr (BITS == 4) {
            const int byte = kk >> 1;
            const int sl = byte / (4 * L), t = (byte % (4 * L)) / L, j = (byte % L) / 4;
            const int i = sl * KTI + 2 * j;
            stage[frag_idx(i, nb, lb + t, NB, lw, paired)] =
                make_uint2(pack_pair(pc[p][0], pc[p][4]), pack_pair(pc[p][1], pc[p][5]));
            stage[frag_idx(i + 1, nb, lb + t, NB, lw, paired)] =
                make_uint2(pack_pair(pc[p][2], pc[p][6]), pack_pair(pc[p][3], pc[p][7]));
        } else {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int byte = kk + 4 * h;
                const int sl = byte / (4 * L), t = (byte % (4 * L)) / L, j = (byte % L) / 4;
                const int i = sl * KTI + j;
                stage[frag_idx(i, nb, lb + t, NB, lw, paired)] =
                    make_uint2(pack_pair(pc[p][4 * h], pc[p][4 * h + 2]), pack_pair(pc[p][4 * h + 1], pc[p][4 * h + 3]));
            }
        }
    }
}

// 16 bytes from global memory; CG: through L2 only (data another CTA of the same grid
// may have written since this SM last read it).
template <bool CG>
Q4_DEVINL uint4 ld_x16(const void *p) {
    if constexpr (CG) {
        uint4 r;
        asm volatile("ld.global.cg.v4.u32 {%0,%1,%2,%3}, [%4];"
                     : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p) : "memory");
        return r;
    } else {
        return *reinterpret_cast<const uint4 *>(p);
    }
}

// 8 activations from index idx of x (fp32, or bf16 widened exactly to fp32).
template <bool XBF16, bool CG = false>
Q4_DEVINL void load_x8(const void *x, int64_t idx, float (&v)[8]) {
    if constexpr (XBF16) {
        const uint4 b = ld_x16<CG>(reinterpret_cast<const uint16_t *>(x) + idx);
        const uint32_t w[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            v[2 * q] = __uint_as_float(w[q] << 16);
            v[2 * q + 1] = __uint_as_float(w[q] & 0xffff0000u);
        }
    } else {
        const uint4 a = ld_x16<CG>(reinterpret_cast<const float *>(x) + idx);
        const uint4 b = ld_x16<CG>(reinterpret_cast<const float *>(x) + idx + 4);
        v[0] = __uint_as_float(a.x); v[1] = __uint_as_float(a.y); v[2] = __uint_as_float(a.z);
        v[3] = __uint_as_float(a.w); v[4] = __uint_as_float(b.x); v[5] = __uint_as_float(b.y);
        v[6] = __uint_as_float(b.z); v[7] = __uint_as_float(b.w);
    }
}

// ---- decode of the packed codes ------------------------------------------------------
// bf16x2 a * b + c, rounded to nearest (exact here: small integers).
Q4_DEVINL uint32_t bfma2(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t d;
    asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}
constexpr uint32_t kBf16One2 = 0x3f803f80u;  // (1.0, 1.0)
// int4: nibbles 0..3 and 16..19 of v (u = code + 8) -> the bf16 pair of codes:
// (128 + u) * 1 - 136.
Q4_DEVINL uint32_t codes4(uint32_t v) {
    return bfma2(and_or(v, 0x000f000fu, 0x43004300u), kBf16One2, 0xc308c308u);
}
// int8: bytes 0 and 2 of v (two's complement codes) -> the bf16 pair of codes:
// (128 + (c & 127)) * 1 - (128, or 256 when c < 0).
Q4_DEVINL uint32_t codes8(uint32_t v) {
    return bfma2(and_or(v, 0x007f007fu, 0x43004300u), kBf16One2, and_or(v, 0x00800080u, 0xc300c300u));
}

// A fragment of MMA j of a segment from one lane's words of row g (w0) and row g+8 (w1).
// int4: word j/2 gives two MMAs; nibble pairs (0,4), (1,5) feed MMA 2*(j/2) (slots 2t,
// 2t+1 and 2t+8, 2t+9), pairs (2,6), (3,7) the next one. int8: word j, byte pairs (0,2)
// and (1,3).
template <int BITS, int L>
Q4_DEVINL void unpack_a(uint32_t (&a)[4], const uint32_t (&w0)[L / 4], const uint32_t (&w1)[L / 4], int j) {
    if constexpr (BITS == 4) {
        const uint32_t x0 = w0[j >> 1], x1 = w1[j >> 1];
        const int s = (j & 1) * 8;
        a[0] = codes4(x0 >> s);
        a[1] = codes4(x1 >> s);
        a[2] = codes4(x0 >> (s + 4));
        a[3] = codes4(x1 >> (s + 4));
    } else {
        const uint32_t x0 = w0[j], x1 = w1[j];
        a[0] = codes8(x0);
        a[1] = codes8(x1);
        a[2] = codes8(x0 >> 8);
        a[3] = codes8(x1 >> 8);
    }
}

// D[16x8] (+)= A[16x16] * B[16x8], bf16 inputs, fp32 accumulate.
Q4_DEVINL void mma_bf16(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// D = A * B (a zero accumulator starts a new group sum without clearing registers).
Q4_DEVINL void mma_bf16_z(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%10,%10,%10,%10};"
        : "=f"(c[0]), "=f"(c[1]), "=f"(c[2]), "=f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(0.f));
}

// Physical row (0..7) inside a 16-row tile of MMA row g (and g + 8), chosen so that the
// shared-memory reads of one instruction hit distinct banks under the 128-byte swizzle
// (8 lanes per phase for 16-byte reads, 16 for 8-byte, 32 for 4-byte).
template <int L>
Q4_DEVINL int row_perm(int g) {
    if constexpr (L == 16) return (g >> 1) + 4 * (g & 1);
    else if constexpr (L == 8) return 2 * (g & 3) + (g >> 2);
    else return g;
}

// L bytes at p (a swizzled position inside a stage, computed once per lane).
template <int L>
Q4_DEVINL void lds_words(uint32_t (&dst)[L / 4], const uint8_t *p) {
    if constexpr (L == 16) {
        const uint4 v = *reinterpret_cast<const uint4 *>(p);
        dst[0] = v.x; dst[1] = v.y; dst[2] = v.z; dst[3] = v.w;
    } else if constexpr (L == 8) {
        const uint2 v = *reinterpret_cast<const uint2 *>(p);
        dst[0] = v.x; dst[1] = v.y;
    } else {
        dst[0] = *reinterpret_cast<const uint32_t *>(p);
    }
}

// B fragment (b0, b1) of MMA i, n8 block nb, from this lane's pieces of the stage.
template <int NB, int LW, bool PAIRED>
Q4_DEVINL void load_b(const uint8_t *frl, int i, int nb, uint4 (&bq)[PAIRED ? NB : 1], uint32_t &b0, uint32_t &b1) {
    if constexpr (PAIRED) {
        if ((i & 1) == 0) bq[nb] = *reinterpret_cast<const uint4 *>(frl + ((i >> 1) * NB + nb) * LW * 16);
        b0 = (i & 1) ? bq[nb].z : bq[nb].x;
        b1 = (i & 1) ? bq[nb].w : bq[nb].y;
    } else {
        const uint2 bb = *reinterpret_cast<const uint2 *>(frl + (i * NB + nb) * LW * 8);
        b0 = bb.x;
        b1 = bb.y;
    }
}

// The group sums of one stage when its group structure is known at compile time.
// GPS >= 1: the stage holds GPS whole groups; GPS == 0: the stage lies inside one group.
// Every group starts with a zero-accumulator MMA; with one n8 block each group has its
// own accumulators (independent chains), otherwise one set is flushed and reused. A flush
// multiplies the fp32 sums by the group's fp32 scale (s0p / s1p: scales of the stage's
// first group for rows g and g + 8) into the totals acc.
// frl: this lane's pieces of the stage. FULL: every segment of the stage is valid;
// otherwise the first nsl are (whole groups when GPS >= 1).
template <int BITS, int L, int NB, int LW, int GPS, bool FULL>
Q4_DEVINL void stage_fixed(const uint32_t (&A0)[kTileBytes / (4 * L)][L / 4],
                           const uint32_t (&A1)[kTileBytes / (4 * L)][L / 4], const uint8_t *frl,
                           const float *s0p, const float *s1p, int nsl, float (&acc)[NB][4]) {
    constexpr int SPS = kTileBytes / (4 * L);
    constexpr int KTI = BITS == 4 ? L / 2 : L / 4;
    constexpr int KTS = SPS * KTI;
    constexpr int NG = GPS > 0 ? GPS : 1;  // groups per stage
    constexpr int IPG = KTS / NG;          // MMAs per group
    constexpr bool PAIRED = NB <= 2;
    constexpr int CH = NB == 1 ? (NG < 4 ? NG : 4) : 1;  // accumulator sets (groups rotate over them)
    float c[CH][NB][4];
    uint4 bq[PAIRED ? NB : 1];
    auto flush = [&](int q, float (&cc)[NB][4]) {
        const float s0 = s0p[q], s1 = s1p[q];
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) {
            acc[nb][0] = fmaf(s0, cc[nb][0], acc[nb][0]);
            acc[nb][1] = fmaf(s0, cc[nb][1], acc[nb][1]);
            acc[nb][2] = fmaf(s1, cc[nb][2], acc[nb][2]);
            acc[nb][3] = fmaf(s1, cc[nb][3], acc[nb][3]);
        }
    };
#pragma unroll
    for (int i = 0; i < KTS; ++i) {
        const int sl = i / KTI, j = i % KTI, q = i / IPG, ch = CH > 1 ? q % CH : 0;
        if (FULL || sl < nsl) {
            // a set that an earlier group of this stage used: that group's sums go out first
            if (CH > 1 && i % IPG == 0 && q >= CH) flush(q - CH, c[ch]);
            uint32_t af[4];
            unpack_a<BITS, L>(af, A0[sl], A1[sl], j);
#pragma unroll
            for (int nb = 0; nb < NB; ++nb) {
                uint32_t b0, b1;
                load_b<NB, LW, PAIRED>(frl, i, nb, bq, b0, b1);
                if (i % IPG == 0)
                    mma_bf16_z(c[ch][nb], af, b0, b1);
                else
                    mma_bf16(c[ch][nb], af, b0, b1);
            }
            if constexpr (CH == 1) {
                // one accumulator set: flush at the end of each group (GPS == 0: at the
                // last valid segment of the stage)
                const bool last = GPS > 0 ? (i % IPG == IPG - 1)
                                          : (FULL ? i == KTS - 1 : (j == KTI - 1 && sl == nsl - 1));
                if (last) flush(q, c[0]);
            }
        }
    }
    if constexpr (CH > 1) {
        // each set still holds the last valid group that used it
        auto valid = [&](int q) { return q < NG && (FULL || q * (SPS / NG) < nsl); };
#pragma unroll
        for (int q = 0; q < NG; ++q)
            if (valid(q) && !valid(q + CH)) flush(q, c[q % CH]);
    }
}



// ======================================================================================
// One row of x: a per-stage choice between exact integer digits and exact bf16 pieces
// ======================================================================================
// When the activations of a 128-byte stage span a dynamic range of at most 2^21 (every
// nonzero |x| >= 2^(E - 21), where max |x| < 2^E), each one is written as the 40-bit
// fixed-point integer X = rint(x * 2^(38 - E)), split into five balanced base-256 digits
// (one int8 MMA column each), and the codes enter the tensor core as int8 (int8 codes as
// stored; int4 nibbles as 16 * code). Every product and every sum of a scale group is then
// an exact integer; the only rounding of x is X's, at most 2^(E - 39) = 2^-18 of the
// element's own magnitude. Stages with a wider range (or extreme exponents) use the bf16
// pieces instead (exact products for any finite x). Both are integrated per lane into two
// fp32 sums (rows g and g + 8 of the warp's tile).
//
// Slot of one stage: the B fragments (either format: the same size) and a header.
//   pieces: k16 MMAs x 16 lanes stored x 8 bytes, columns (hi, mid, lo, 0) [P = 3] or
//           (x, 0, 0, 0) [P = 1]
//   digits: k32 MMAs x 32 lanes x 8 bytes, column c holds digit 4 - c, columns 5-7 zero
//   header: int mode (1 = digits), float f = 2^(E - 38) (x 2^-4 for int4, whose A operand
//           is 16 * code)
template <int BITS>
__host__ __device__ constexpr int slot1_data() { return BITS == 4 ? 2048 : 1024; }
template <int BITS>
__host__ __device__ constexpr int slot1_bytes() { return slot1_data<BITS>() + 16; }

Q4_DEVINL float pow2i(int e) { return __int_as_float((e + 127) << 23); }  // 2^e, e in [-126, 127]

// Smallest E with max|x| < 2^E from the bits of max|x| (> 0, finite).
Q4_DEVINL int exp_above(uint32_t mx) {
    const int be = (int)(mx >> 23);
    if (be > 0) return be - 126;
    return (32 - __clz((int)mx)) - 149;  // subnormal: mx * 2^-149 with mx < 2^23
}

// Decision for a stage from the bits of its max |x| and of its smallest nonzero |x|
// (0x7f800000 when every x is 0): digits when the range condition holds and E leaves the
// scale factors normal; *E_out is E (0 for an all-zero stage).
Q4_DEVINL bool digits_ok(uint32_t mx, uint32_t mn, int *E_out) {
    if (mx >= 0x7f800000u) return false;  // Inf or NaN: the pieces carry them
    if (mx == 0) {
        *E_out = 0;
        return true;
    }
    const int E = exp_above(mx);
    *E_out = E;
    if (E < -60 || E > 100) return false;
    const int te = E - 21;  // threshold 2^te
    const uint32_t thr = te >= -126 ? (uint32_t)(te + 127) << 23 : (te >= -149 ? 1u << (te + 149) : 0u);
    return mn >= thr;
}

// Balanced base-256 digits of X = rint(x * 2^(38 - E)), |X| < 2^38: returns the 64-bit
// word whose bytes 0..4 are the digits (two's complement int8), digit p of weight 256^p.
Q4_DEVINL uint64_t digits5(float x, int E) {
    const int sh = 38 - E;  // 38 - E in [-62, 98]: two exact power-of-two steps
    const int s1 = sh > 64 ? 64 : sh;
    const float v = (x * pow2i(s1)) * pow2i(sh - s1);
    const long long X = __float2ll_rn(v);
    return ((uint64_t)X + 0x8080808080ull) ^ 0x8080808080ull;
}

// out[p] = byte p of (a, b, c, d), in that order.
Q4_DEVINL void bytes_transpose4(uint32_t a, uint32_t b, uint32_t c, uint32_t d, uint32_t (&out)[4]) {
    const uint32_t t0 = prmt(a, b, 0x5140u), t1 = prmt(a, b, 0x7362u);
    const uint32_t t2 = prmt(c, d, 0x5140u), t3 = prmt(c, d, 0x7362u);
    out[0] = prmt(t0, t2, 0x5410u);
    out[1] = prmt(t0, t2, 0x7632u);
    out[2] = prmt(t1, t3, 0x5410u);
    out[3] = prmt(t1, t3, 0x7632u);
}
// Byte 0 of each of a, b, c, d, in that order.
Q4_DEVINL uint32_t bytes0(uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    return prmt(prmt(a, b, 0x0040u), prmt(c, d, 0x0040u), 0x5410u);
}

// Digit-format B fragments of 8 consecutive k (offset kk in the stage, a multiple of 8):
// one lane slice of one k32 MMA. int4: b0 = the even k of the word, b1 = the odd k (the
// low and high nibbles of its bytes); int8: b0 = k 0..3, b1 = k 4..7.
template <int BITS, int L>
Q4_DEVINL void digits_unit(uint2 *slot, int kk, const float (&v)[8], int E) {
    constexpr int KTID = BITS == 4 ? L / 4 : L / 8;  // k32 MMAs per segment
    const int byte = BITS == 4 ? (kk >> 1) : kk;
    const int sl = byte / (4 * L), t = (byte % (4 * L)) / L;
    const int j = BITS == 4 ? (byte % L) / 4 : (byte % L) / 8;
    const int i = sl * KTID + j;
    uint64_t D[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) D[q] = digits5(v[q], E);
    const int q0[4] = {BITS == 4 ? 0 : 0, BITS == 4 ? 2 : 1, BITS == 4 ? 4 : 2, BITS == 4 ? 6 : 3};
    const int o = BITS == 4 ? 1 : 4;  // b1 takes the values q0[] + o
    uint32_t T0[4], T1[4];
    bytes_transpose4((uint32_t)D[q0[0]], (uint32_t)D[q0[1]], (uint32_t)D[q0[2]], (uint32_t)D[q0[3]], T0);
    bytes_transpose4((uint32_t)D[q0[0] + o], (uint32_t)D[q0[1] + o], (uint32_t)D[q0[2] + o], (uint32_t)D[q0[3] + o],
                     T1);
    const uint32_t h0 = bytes0((uint32_t)(D[q0[0]] >> 32), (uint32_t)(D[q0[1]] >> 32), (uint32_t)(D[q0[2]] >> 32),
                               (uint32_t)(D[q0[3]] >> 32));
    const uint32_t h1 = bytes0((uint32_t)(D[q0[0] + o] >> 32), (uint32_t)(D[q0[1] + o] >> 32),
                               (uint32_t)(D[q0[2] + o] >> 32), (uint32_t)(D[q0[3] + o] >> 32));
    auto at = [&](int col) -> uint2 & { return slot[frag_idx(i, 0, 4 * col + t, 1, 32, true)]; };
    at(0) = make_uint2(h0, h1);  // digit 4
#pragma unroll
    for (int p = 3; p >= 0; --p) at(4 - p) = make_uint2(T0[p], T1[p]);
#pragma unroll
    for (int col = 5; col < 8; ++col) at(col) = make_uint2(0u, 0u);
}

// Piece-format B fragments of 8 consecutive k, every stored column written (the columns
// no piece uses are zero).
template <int BITS, int L>
Q4_DEVINL void pieces_unit(uint2 *slot, int kk, const float (&v)[8], int P) {
    frag_unit<BITS, L>(slot, kk, 0, v, P, 4, 1, 16, true);
    float z[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) z[q] = 0.f;
    for (int vm = 1; vm * P < 4; ++vm) frag_unit<BITS, L>(slot, kk, vm, z, P, 4, 1, 16, true);
}

// A fragment of k32 int8 MMA j of a segment (digits format) from one lane's words of row
// g (w0) and row g + 8 (w1). int4: byte (u_hi << 4 | u_lo), u = code + 8: (u << 4) ^ 0x80
// is the int8 16 * code.
template <int BITS, int L>
Q4_DEVINL void unpack_a8(uint32_t (&a)[4], const uint32_t (&w0)[L / 4], const uint32_t (&w1)[L / 4], int j) {
    if constexpr (BITS == 4) {
        const uint32_t x0 = w0[j], x1 = w1[j];
        a[0] = ((x0 << 4) & 0xF0F0F0F0u) ^ 0x80808080u;  // even k of row g
        a[1] = ((x1 << 4) & 0xF0F0F0F0u) ^ 0x80808080u;  // even k of row g + 8
        a[2] = (x0 & 0xF0F0F0F0u) ^ 0x80808080u;         // odd k of row g
        a[3] = (x1 & 0xF0F0F0F0u) ^ 0x80808080u;         // odd k of row g + 8
    } else {
        a[0] = w0[2 * j];
        a[1] = w1[2 * j];
        a[2] = w0[2 * j + 1];
        a[3] = w1[2 * j + 1];
    }
}

// One stage of one row of x in the pieces format: the group sums of the two piece columns
// this lane holds, scaled by the group's fp32 scale, go into y0 (row g) and y1 (row g + 8).
template <int BITS, int L, int GPS, bool FULL>
Q4_DEVINL void stage1_pieces(const uint32_t (&A0)[kTileBytes / (4 * L)][L / 4],
                             const uint32_t (&A1)[kTileBytes / (4 * L)][L / 4], const uint8_t *slot, int lane,
                             const float *s0p, const float *s1p, int nsl, float &y0, float &y1) {
    constexpr int SPS = kTileBytes / (4 * L);
    constexpr int KTI = BITS == 4 ? L / 2 : L / 4;
    constexpr int KTS = SPS * KTI;
    constexpr int NG = GPS > 0 ? GPS : 1;
    constexpr int IPG = KTS / NG;
    constexpr int CH = NG < 4 ? NG : 4;
    const uint8_t *frl = slot + (lane & 15) * 16;
    // lanes 16-31 read the fragments of lanes 0-15: their columns (4-7) repeat columns
    // 0-3 and must not be counted
    const bool own = (lane & 2) == 0;
    float c[CH][4];
    uint4 bq[1];
    auto flush = [&](int q, float (&cc)[4]) {
        if (own) {
            y0 = fmaf(s0p[q], cc[0] + cc[1], y0);
            y1 = fmaf(s1p[q], cc[2] + cc[3], y1);
        }
    };
    auto valid = [&](int q) { return q < NG && (FULL || q * (SPS / NG) < nsl); };
#pragma unroll
    for (int i = 0; i < KTS; ++i) {
        const int sl = i / KTI, j = i % KTI, q = i / IPG, ch = q % CH;
        if (FULL || sl < nsl) {
            if (CH > 1 && i % IPG == 0 && q >= CH) flush(q - CH, c[ch]);
            uint32_t af[4];
            unpack_a<BITS, L>(af, A0[sl], A1[sl], j);
            uint32_t b0, b1;
            load_b<1, 16, true>(frl, i, 0, bq, b0, b1);
            if (i % IPG == 0)
                mma_bf16_z(c[ch], af, b0, b1);
            else
                mma_bf16(c[ch], af, b0, b1);
            if constexpr (CH == 1) {
                const bool last = GPS > 0 ? (i % IPG == IPG - 1)
                                          : (FULL ? i == KTS - 1 : (j == KTI - 1 && sl == nsl - 1));
                if (last) flush(q, c[0]);
            }
        }
    }
    if constexpr (CH > 1) {
#pragma unroll
        for (int q = 0; q < NG; ++q)
            if (valid(q) && !valid(q + CH)) flush(q, c[q % CH]);
    }
}

// The same stage in the digits format: exact int32 group sums; a lane's column pair
// (digits d, d - 1) combines exactly as 256 * c0 + c1 and is scaled by the group's scale
// times fl (2^(E - 38), the lane's pair weight 256^(3 - 2t) and the int4 factor 2^-4).
template <int BITS, int L, int GPS, bool FULL>
Q4_DEVINL void stage1_digits(const uint32_t (&A0)[kTileBytes / (4 * L)][L / 4],
                             const uint32_t (&A1)[kTileBytes / (4 * L)][L / 4], const uint8_t *slot, int lane,
                             const float *s0p, const float *s1p, int nsl, float fl, float &y0, float &y1) {
    constexpr int SPS = kTileBytes / (4 * L);
    constexpr int KTI = BITS == 4 ? L / 4 : L / 8;  // k32 MMAs per segment
    constexpr int KTS = SPS * KTI;
    constexpr int NG = GPS > 0 ? GPS : 1;
    constexpr int IPG = KTS / NG;
    constexpr int CH = NG < 4 ? NG : 4;
    const uint8_t *frl = slot + lane * 16;
    int c[CH][4];
    uint4 bq[1];
    auto flush = [&](int q, int (&cc)[4]) {
        const int p0 = cc[0] * 256 + cc[1], p1 = cc[2] * 256 + cc[3];
        y0 = fmaf(s0p[q] * fl, __int2float_rn(p0), y0);
        y1 = fmaf(s1p[q] * fl, __int2float_rn(p1), y1);
    };
    auto valid = [&](int q) { return q < NG && (FULL || q * (SPS / NG) < nsl); };
#pragma unroll
    for (int i = 0; i < KTS; ++i) {
        const int sl = i / KTI, j = i % KTI, q = i / IPG, ch = q % CH;
        if (FULL || sl < nsl) {
            if (CH > 1 && i % IPG == 0 && q >= CH) flush(q - CH, c[ch]);
            uint32_t af[4];
            unpack_a8<BITS, L>(af, A0[sl], A1[sl], j);
            uint32_t b0, b1;
            load_b<1, 32, true>(frl, i, 0, bq, b0, b1);
            if (i % IPG == 0)
                mma_s8_16832_z(c[ch], af, b0, b1);
            else
                mma_s8_16832(c[ch], af, b0, b1);
            if constexpr (CH == 1) {
                const bool last = GPS > 0 ? (i % IPG == IPG - 1)
                                          : (FULL ? i == KTS - 1 : (j == KTI - 1 && sl == nsl - 1));
                if (last) flush(q, c[0]);
            }
        }
    }
    if constexpr (CH > 1) {
#pragma unroll
        for (int q = 0; q < NG; ++q)
            if (valid(q) && !valid(q + CH)) flush(q, c[q % CH]);
    }
}

// Builds the slot of one stage from the calling lane's 8 activations v (k = 8 * lane + q
// of the stage; zeros past K and in lanes past the stage): the warp decides the format
// together and writes every byte of the slot (header by lane 0).
template <int BITS, int L>
Q4_DEVINL void build_slot1_v(uint8_t *slot, const float (&v)[8], int P, int lane) {
    constexpr int STAGEK = kTileBytes * 8 / BITS;
    constexpr int LANES = STAGEK / 8;
    const int kk = 8 * lane;
    uint32_t mx = 0, mn = 0x7f800000u;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        const uint32_t a = __float_as_uint(v[q]) & 0x7fffffffu;
        mx = max(mx, a);
        if (a != 0) mn = min(mn, a);
    }
    mx = __reduce_max_sync(0xffffffffu, mx);
    mn = __reduce_min_sync(0xffffffffu, mn);
    int E = 0;
    const bool dig = digits_ok(mx, mn, &E);
    uint2 *s2 = reinterpret_cast<uint2 *>(slot);
    if (lane < LANES) {
        if (dig)
            digits_unit<BITS, L>(s2, kk, v, E);
        else
            pieces_unit<BITS, L>(s2, kk, v, P);
    }
    if (lane == 0) {
        int *h = reinterpret_cast<int *>(slot + slot1_data<BITS>());
        h[0] = dig ? 1 : 0;
        h[1] = E;
    }
}

// The same from x[k0, k0 + STAGEK) in global memory (zeros past K): the calling warp's
// lanes load 8 k each (all 32 for int4, 16 for int8).
template <int BITS, int L, bool XBF16, bool CG>
Q4_DEVINL void build_slot1(uint8_t *slot, const void *x, int k0, int K, int P, int lane) {
    constexpr int STAGEK = kTileBytes * 8 / BITS;
    constexpr int LANES = STAGEK / 8;
    const int kk = 8 * lane;
    float v[8];
    if (lane < LANES && k0 + kk < K) {
        load_x8<XBF16, CG>(x, k0 + kk, v);
    } else {
#pragma unroll
        for (int q = 0; q < 8; ++q) v[q] = 0.f;
    }
    build_slot1_v<BITS, L>(slot, v, P, lane);
}

// The lane's multiplier of the digits format: 2^(E - 38) times its column pair's weight
// 256^(3 - 2t) (t = lane & 3; pairs (4, 3), (2, 1), (0, -)), times 2^-4 for int4.
template <int BITS>
Q4_DEVINL float digit_lane_factor(int E, int t) {
    return pow2i(E - 38 + 24 - 16 * t - (BITS == 4 ? 4 : 0));
}

}  // namespace gm
}  // namespace q4
