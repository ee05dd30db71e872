// gemv.cu -- fused unpack -> dequant -> GEMV for decode (x in chunks of 16 rows).
//
// y[m][n] = sum_k x[m][k] * w'[n][k], w' = code * scale (pack()/unpack() of the
// "量化推理" page; the QuantizedMatmul of "Huit bits, puis quatre", which reads the
// codes in generation products, where one waits on memory). The packed weights are the
// whole cost, so the kernel is built around streaming them with as few instructions per
// byte as possible.
//
// Arithmetic: exact integer dot products on the tensor cores (warp-level mma.sync
// m16n8k32, s8 x s8 -> s32).
//   A = 16 weight rows x 32 k of codes as int8: int8 codes as they are stored; int4
//       nibbles u = code + 8 become the byte 16 * code with one mask-and-xor (high
//       nibble) or shift-mask-xor (low nibble), so a 32-bit word of 8 codes costs three
//       logic instructions. The factor 16 is an exact power of two folded in at the end.
//   B = 32 k x 8 columns of activation digits: each activation row m is written, per
//       block of k, as the 32-bit fixed-point value X = rint(x * 2^(30-E)) (E chosen so
//       that max|x| over the block is below 2^E) and X is split into four balanced
//       base-256 digits in [-128, 127]; one B column per digit.
//   C = int32, exact: the products and their sums within a scale group are integers.
// When a scale group ends (or a 128-byte stage ends) each lane combines its two digit
// columns 256*c0 + c1 (still exact), converts once to fp32, multiplies by the group's
// fp32 scale and accumulates in fp32; the block's 2^(E-30) (and 2^16 for the high digit
// pair) is applied exactly when the k-block ends. The only roundings are the fixed-point
// activation (2^-31 of the block maximum) and the fp32 sums of the group results.
//
// Structure (one wave: up to two CTAs per SM, a thread-block cluster of CS CTAs splits K):
//   a producer warp issues, per stage, one 2D TMA load of a 128-row x 128-byte tile of
//   the payload (128-byte swizzle) into a shared-memory ring guarded by full/empty
//   mbarriers, and loads each k-block's scales into double-buffered shared memory with
//   asynchronous copies (16 bytes wide when the rows of scales allow) one block ahead;
//   eight consumer warps decode and multiply.
//   One activation row (the decode case): the consumers build the digits of their CTA's
//   K range into shared memory while the first payload tiles are in flight; there is no
//   second kernel and no workspace.
//   Several rows: gemv_prep writes the digits once into the caller's workspace, in MMA
//   order, and the stream kernel (its programmatic dependent) copies each stage's tile
//   with a bulk copy into a second ring; the payload loads start before gemv_prep ends.
// Inside a group the order of k is permuted so that a lane builds its A fragment from its
// own shared-memory words; the digits use the same permutation. Rows are permuted inside
// each 16-row tile so those reads are free of bank conflicts. The CS partial sums of a
// cluster meet in distributed shared memory in fixed rank order, so results do not depend
// on timing. Every wait is bounded; one that gives up sets Q4_STATUS_TIMEOUT.
#include <cuda.h>  // CUtensorMap and its enums (the encoder is fetched at run time)

#include "common.cuh"
#include "kernels.h"

namespace q4 {

namespace {

constexpr int kConsumers = 8;                      // consumer warps = 16-row tiles per CTA
constexpr int kConsumerThreads = 32 * kConsumers;
constexpr int kThreads = kConsumerThreads + 32;    // + 1 producer warp (the last warp)
constexpr int kRowsPerCta = 16 * kConsumers;       // 128
constexpr int kTileBytes = 128;                    // bytes of a weight row per stage
constexpr int kPayloadBytes = kTileBytes * kRowsPerCta;  // 16 KB of codes per stage
constexpr int kMaxStages = 6;
constexpr int kGroupsPerBlock = 8;                 // scale groups per k-block (target)
constexpr int kBlockK = 1024;                      // at most k per k-block
constexpr int kSG = 12;                            // scale slots per row per k-block (<= 9 used,
                                                   // + up to 3 to keep 16-byte copies aligned)
constexpr int kMaxLocalBlocks = 40;                // k-blocks one CTA may touch (in-kernel digits)
constexpr int kFragCap = 32768;                    // in-kernel digit bytes (4 per k)
constexpr int kSmemBudget = 115200;                // two CTAs per SM
constexpr int kRedBytes = kRowsPerCta * 16 * 4;    // cluster partial sums, aliased on the ring

struct GemvArgs {
    const float *scales;
    const void *x;
    float *y;
    uint32_t *status;
    uint8_t *frag;        // workspace digits: [mc][stage][fslot_bytes] (several rows of x)
    int *ebexp;           // workspace exponents: [mc*16 + m][n_eb]
    int M, N, K;
    int segs;             // segments per weight row
    int spg;              // segments per scale group
    int scales_per_row;   // K / group
    int CS;               // CTAs per cluster = K splits
    int stages_total;     // 128-byte tiles per weight row (last may be partial)
    int stages_per_cta;
    int ebs;              // stages per k-block (exponent and scale block)
    int n_eb;
    int lw;               // digit lanes per (MMA, n8 block): 16 for one row of x, else 32
    int NB;               // n8 blocks per 16-row chunk of x (2 rows of x per block)
    int paired;           // digits of two consecutive MMAs interleaved (16-byte reads)
    int nst_ring;         // ring depth
    int fslot_bytes;      // digit bytes of one stage
};

// ---- small PTX helpers for clusters --------------------------------------------------
Q4_DEVINL void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
Q4_DEVINL float ld_dsmem_f32(const float *local_smem_ptr, uint32_t rank) {
    uint32_t a = (uint32_t)__cvta_generic_to_shared(local_smem_ptr), r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(rank));
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(r));
    return v;
}
Q4_DEVINL void bulk_copy_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// ---- activation digits --------------------------------------------------------------
Q4_DEVINL float pow2(int e) { return __int_as_float((e + 127) << 23); }  // 2^e, e in [-126, 127]

// v * 2^e in two exact power-of-two steps (e may leave [-126, 127]); one rounding at most,
// and only when the result is subnormal.
Q4_DEVINL float scale2(float v, int e) {
    const int e1 = min(max(e, -126), 127);
    const int e2 = min(max(e - e1, -126), 127);
    return (v * pow2(e1)) * pow2(e2);
}

// E such that every |x| of a block is below 2^E, from the bits of the block's max |x|;
// 0 for an all-zero (or non-finite) block.
Q4_DEVINL int block_exp(uint32_t mx) {
    if (mx == 0 || mx >= 0x7f800000u) return 0;
    const int be = (int)(mx >> 23);
    if (be > 0) return be - 126;
    return (32 - __clz((int)mx)) - 149;  // subnormal: mx * 2^-149 with mx < 2^23
}

// Balanced base-256 digits of X = rint(v * 2^(30-E)) (|X| < 2^30), packed with the least
// significant digit in byte 0: X = sum_p digit_p * 256^p, every digit in [-128, 127].
// (X + 0x808080) has unsigned low bytes b_p; digit_p = b_p - 128, i.e. b_p ^ 0x80.
Q4_DEVINL uint32_t digits4(float v, float f1, float f2) {
    const int X = __float2int_rn((v * f1) * f2);
    return (uint32_t)(X + 0x00808080) ^ 0x00808080u;
}

// out[p] = byte p of (a, b, c, d), in that order.
Q4_DEVINL void transpose4(uint32_t a, uint32_t b, uint32_t c, uint32_t d, uint32_t (&out)[4]) {
    const uint32_t t0 = prmt(a, b, 0x5140u), t1 = prmt(a, b, 0x7362u);
    const uint32_t t2 = prmt(c, d, 0x5140u), t3 = prmt(c, d, 0x7362u);
    out[0] = prmt(t0, t2, 0x5410u);
    out[1] = prmt(t0, t2, 0x7632u);
    out[2] = prmt(t1, t3, 0x5410u);
    out[3] = prmt(t1, t3, 0x7632u);
}

// Index (uint2 units) of the B fragment of MMA i of a stage, n8 block nb, lane.
Q4_DEVINL int frag_idx(int i, int nb, int lane, int NB, int lw, bool paired) {
    return paired ? ((((i >> 1) * NB + nb) * lw + lane) << 1) + (i & 1) : (i * NB + nb) * lw + lane;
}

// The B fragments of 8 consecutive k (offset kk inside the stage, a multiple of 8) of
// activation row m of a 16-row chunk. Column 4h + (3 - p) of n8 block m/2 (h = m % 2)
// holds digit p, so a lane's accumulator pair (c0, c1) is (digit 3, digit 2) for t even
// and (digit 1, digit 0) for t odd: 256 * c0 + c1 is the high / low half of the sum.
// k-slots of the MMA (PTX m16n8k32 layout) map onto memory k as the lane's A words do:
// int4: b0 = the even k of the word, b1 = the odd k; int8: b0 = k 0..3, b1 = k 4..7.
template <int BITS, int L>
Q4_DEVINL void frag_unit(uint2 *stage, int kk, int m, const float (&v)[8], float f1, float f2, int NB,
                         int lw, bool paired) {
    constexpr int KTI = BITS == 4 ? L / 4 : L / 8;  // MMAs per segment
    const int byte = BITS == 4 ? (kk >> 1) : kk;
    const int sl = byte / (4 * L), t = (byte % (4 * L)) / L;
    const int j = (byte % L) / (BITS == 4 ? 4 : 8);
    const int i = sl * KTI + j;
    uint32_t D[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) D[q] = digits4(v[q], f1, f2);
    uint32_t T0[4], T1[4];
    if constexpr (BITS == 4) {
        transpose4(D[0], D[2], D[4], D[6], T0);
        transpose4(D[1], D[3], D[5], D[7], T1);
    } else {
        transpose4(D[0], D[1], D[2], D[3], T0);
        transpose4(D[4], D[5], D[6], D[7], T1);
    }
    const int nb = m >> 1, h = m & 1;
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        const int lane = 16 * h + 4 * (3 - p) + t;
        stage[frag_idx(i, nb, lane, NB, lw, paired)] = make_uint2(T0[p], T1[p]);
    }
}

template <bool XBF16>
Q4_DEVINL void load_x8(const void *x, int64_t idx, float (&v)[8]) {
    if constexpr (XBF16) {
        const uint4 b = *reinterpret_cast<const uint4 *>(reinterpret_cast<const uint16_t *>(x) + idx);
        const uint32_t w[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            v[2 * q] = __uint_as_float(w[q] << 16);
            v[2 * q + 1] = __uint_as_float(w[q] & 0xffff0000u);
        }
    } else {
        const float4 a = *reinterpret_cast<const float4 *>(reinterpret_cast<const float *>(x) + idx);
        const float4 b = *reinterpret_cast<const float4 *>(reinterpret_cast<const float *>(x) + idx + 4);
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
        v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    }
}

Q4_DEVINL uint32_t absmax8(const float (&v)[8]) {
    uint32_t m = 0;
#pragma unroll
    for (int q = 0; q < 8; ++q) m = max(m, __float_as_uint(v[q]) & 0x7fffffffu);
    return m;
}

// One CTA per (k-block eb, 16-row chunk mc of x): the block exponent of every activation
// row, then the digits of the block in MMA order (several rows of x).
template <int BITS, int L, bool XBF16>
__global__ void __launch_bounds__(256) gemv_prep(const GemvArgs a) {
    grid_dep_launch();
    grid_dep_wait();  // x may be the output of the kernel before this one
    constexpr int STAGEK = kTileBytes * 8 / BITS;
    __shared__ int e_sh[16];
    const int eb = blockIdx.x, mc = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int mcnt = min(16, a.M - mc * 16);
    const int k0 = eb * a.ebs * STAGEK;
    const int k1 = min(a.K, k0 + a.ebs * STAGEK);
    const int nu = (k1 - k0) / 8;  // 8-k units in the block (at most 128)
    for (int ml = warp; ml < 16; ml += 8) {
        uint32_t mx = 0;
        if (ml < mcnt) {
            const int64_t rowb = (int64_t)(mc * 16 + ml) * a.K + k0;
#pragma unroll
            for (int r = 0; r < kBlockK / 256; ++r) {
                const int u = lane + 32 * r;
                if (u < nu) {
                    float v[8];
                    load_x8<XBF16>(a.x, rowb + 8 * u, v);
                    mx = max(mx, absmax8(v));
                }
            }
        }
        mx = __reduce_max_sync(0xffffffffu, mx);
        if (lane == 0) {
            const int E = block_exp(mx);
            e_sh[ml] = E;
            a.ebexp[(int64_t)(mc * 16 + ml) * a.n_eb + eb] = E;
        }
    }
    __syncthreads();
    uint2 *fbase = reinterpret_cast<uint2 *>(a.frag) + (size_t)mc * a.stages_total * (a.fslot_bytes / 8);
    for (int it = threadIdx.x; it < nu * mcnt; it += blockDim.x) {
        const int ml = it / nu, u = it - ml * nu;
        const int k = k0 + 8 * u;
        float v[8];
        load_x8<XBF16>(a.x, (int64_t)(mc * 16 + ml) * a.K + k, v);
        const int sh = 30 - e_sh[ml];
        const int e1 = min(max(sh, -126), 127);
        const float f1 = pow2(e1), f2 = pow2(min(max(sh - e1, -126), 127));
        const int s = k / STAGEK;
        frag_unit<BITS, L>(fbase + (size_t)s * (a.fslot_bytes / 8), k - s * STAGEK, ml, v, f1, f2, a.NB, a.lw,
                           a.paired != 0);
    }
}

// ---- decode of the packed codes ------------------------------------------------------
// A fragment of MMA j of a segment from one lane's words of row g (w0) and row g+8 (w1).
template <int BITS, int L>
Q4_DEVINL void unpack_a(uint32_t (&a)[4], const uint32_t (&w0)[L / 4], const uint32_t (&w1)[L / 4], int j) {
    if constexpr (BITS == 4) {
        // byte (u_hi << 4 | u_lo), u = code + 8: (u << 4) ^ 0x80 is the int8 16 * code
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

// The exact group sums of one stage when its group structure is known at compile time.
// GPS >= 1: the stage holds GPS whole groups; GPS == 0: the stage lies inside one group.
// Every group starts with a zero-accumulator MMA; with one n8 block each group has its
// own accumulators (independent chains), otherwise one set is flushed and reused. A flush
// combines the two digit columns (256 * c0 + c1, exact), converts once and applies the
// group's fp32 scale (s0p / s1p: scales of the stage's first group for rows g and g + 8).
// frl: this lane's digits of the stage. FULL: every segment of the stage is valid;
// otherwise the first nsl are (whole groups when GPS >= 1).
template <int BITS, int L, int NB, int LW, int GPS, bool FULL>
Q4_DEVINL void stage_fixed(const uint32_t (&A0)[kTileBytes / (4 * L)][L / 4],
                           const uint32_t (&A1)[kTileBytes / (4 * L)][L / 4], const uint8_t *frl,
                           const float *s0p, const float *s1p, int nsl, float (&y0)[NB], float (&y1)[NB]) {
    constexpr int SPS = kTileBytes / (4 * L);
    constexpr int KTI = BITS == 4 ? L / 4 : L / 8;
    constexpr int KTS = SPS * KTI;
    constexpr int NG = GPS > 0 ? GPS : 1;  // groups per stage
    constexpr int IPG = KTS / NG;          // MMAs per group
    constexpr bool PAIRED = NB <= 2;
    constexpr int CH = NB == 1 ? NG : 1;   // accumulator sets
    int c[CH][NB][4];
    uint4 bq[PAIRED ? NB : 1];
    auto flush = [&](int q, int (&cc)[NB][4]) {
        const float s0 = s0p[q], s1 = s1p[q];
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) {
            const int p0 = cc[nb][0] * 256 + cc[nb][1], p1 = cc[nb][2] * 256 + cc[nb][3];
            y0[nb] = fmaf(s0, __int2float_rn(p0), y0[nb]);
            y1[nb] = fmaf(s1, __int2float_rn(p1), y1[nb]);
        }
    };
#pragma unroll
    for (int i = 0; i < KTS; ++i) {
        const int sl = i / KTI, j = i % KTI, q = i / IPG, ch = CH > 1 ? q : 0;
        if (FULL || sl < nsl) {
            uint32_t af[4];
            unpack_a<BITS, L>(af, A0[sl], A1[sl], j);
#pragma unroll
            for (int nb = 0; nb < NB; ++nb) {
                uint32_t b0, b1;
                if constexpr (PAIRED) {
                    if ((i & 1) == 0) bq[nb] = *reinterpret_cast<const uint4 *>(frl + ((i >> 1) * NB + nb) * LW * 16);
                    b0 = (i & 1) ? bq[nb].z : bq[nb].x;
                    b1 = (i & 1) ? bq[nb].w : bq[nb].y;
                } else {
                    const uint2 bb = *reinterpret_cast<const uint2 *>(frl + (i * NB + nb) * LW * 8);
                    b0 = bb.x;
                    b1 = bb.y;
                }
                if (i % IPG == 0)
                    mma_s8_16832_z(c[ch][nb], af, b0, b1);
                else
                    mma_s8_16832(c[ch][nb], af, b0, b1);
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
#pragma unroll
        for (int q = 0; q < NG; ++q)
            if (FULL || q * (SPS / NG) < nsl) flush(q, c[q]);
    }
}

// INK: one row of x whose digits the consumers build in shared memory (no workspace);
// otherwise the digits come from gemv_prep through a second ring. GPS: groups per stage
// when they divide it, 0 when the stage lies inside one group, -1 for any other group
// size (tracked segment by segment at run time).
template <int BITS, int L, int NB, int GPS, bool INK, bool XBF16>
__global__ void __launch_bounds__(kThreads, 2)
gemv_stream(const GemvArgs a, const __grid_constant__ CUtensorMap tmap) {
    constexpr int SPS = kTileBytes / (4 * L);          // segments per stage
    constexpr int KTI = BITS == 4 ? L / 4 : L / 8;     // MMAs per segment
    constexpr int KTS = SPS * KTI;                     // MMAs per stage (8 int4, 4 int8)
    constexpr int WPT = L / 4;
    constexpr int STAGEK = kTileBytes * 8 / BITS;
    constexpr bool PAIRED = NB <= 2;
    constexpr int LW = INK ? 16 : 32;  // digit lanes stored per (MMA, n8 block)
    static_assert(!INK || NB == 1, "in-kernel digits cover one row of x");
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const int nring = a.nst_ring;
    uint8_t *slots = smem;                                   // codes: nring x 16 KB (1024-aligned)
    uint8_t *fslots = smem + nring * kPayloadBytes;          // digits: ring slots, or the CTA's range
    const int nfrag = INK ? a.stages_per_cta : nring;
    float *scl = reinterpret_cast<float *>(fslots + nfrag * a.fslot_bytes);  // [2][128][kSG]
    uint32_t *mx_sh = reinterpret_cast<uint32_t *>(scl + 2 * kRowsPerCta * kSG);  // [kMaxLocalBlocks]
    uint64_t *full = reinterpret_cast<uint64_t *>(mx_sh + kMaxLocalBlocks);  // codes landed
    uint64_t *empty = full + kMaxStages;                                  // codes copied to registers
    uint64_t *ffull = empty + kMaxStages;                                 // digits landed
    uint64_t *fempty = ffull + kMaxStages;                                // digits no longer read
    uint64_t *sfull = fempty + kMaxStages;
    uint64_t *sempty = sfull + 2;
    float *red = reinterpret_cast<float *>(slots);  // [128][16] partial sums, after the main loop

    // the next call on the stream may start its own prologue (and, when its weights are
    // declared static, stream them) while this grid runs; it waits before reading x
    grid_dep_launch();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int crank = (int)(blockIdx.x % (unsigned)a.CS);
    const int cl = (int)(blockIdx.x / (unsigned)a.CS);
    const int mc = blockIdx.y;
    const int mcnt = min(16, a.M - mc * 16);
    const int st_lo = crank * a.stages_per_cta;
    const int st_hi = min(st_lo + a.stages_per_cta, a.stages_total);
    const int nst = max(st_hi - st_lo, 0);
    const int seg_hi = min(st_hi * SPS, a.segs);
    const int eb_first = st_lo / a.ebs;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kMaxStages; ++i) {
            mbar_init(full + i, 1);
            mbar_init(empty + i, kConsumers);
            mbar_init(ffull + i, 1);
            mbar_init(fempty + i, kConsumers);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(sfull + i, 32);
            mbar_init(sempty + i, kConsumers);
        }
        fence_barrier_init();
    }
    if constexpr (INK) {
        // block maxima of the on-chip digits, zeroed before the barrier that publishes the
        // mbarriers. A CTA's digits fit in kFragCap: at most 32 int4 stages (k-blocks of one
        // or more) or 64 int8 stages (k-blocks of two or more), so at most 33 local k-blocks.
        for (int i = threadIdx.x; i < kMaxLocalBlocks; i += blockDim.x) mx_sh[i] = 0;
    }
    __syncthreads();

    // groups [gA, gA + ng) touched by k-block eb inside this CTA's range
    auto eb_groups = [&](int eb, int &gA, int &ng) {
        const int s0 = max(st_lo, eb * a.ebs), s1 = min(st_hi, (eb + 1) * a.ebs);
        const int sg0 = s0 * SPS, sg1 = min(s1 * SPS, a.segs);
        gA = sg0 / a.spg;
        ng = (sg1 - 1) / a.spg - gA + 1;
    };

    // 16-byte scale copies when every row of scales starts 16-byte aligned
    const bool vec16 = (a.scales_per_row & 3) == 0 && ((uintptr_t)a.scales & 15) == 0;
    bool timed_out = false;
    if (warp == kConsumers) {
        // ---------------- producer warp ----------------
        const uint8_t *fsrc = a.frag + (size_t)mc * a.stages_total * a.fslot_bytes;
        const int primed = min(nst, nring);
        // The first `primed` stages' digits are copied once gemv_prep has finished, so that
        // the codes of those stages stream in meanwhile; `issued` of them have gone out.
        // They go out before any wait on the consumers, who need them to make progress.
        int issued = 0;
        auto issue_primed = [&](int upto) {
            if (issued >= upto) return;
            if (issued == 0) grid_dep_wait();
            if (lane == 0 && !timed_out) {
                const uint32_t fb = (uint32_t)a.fslot_bytes;
                for (int q = issued; q < upto; ++q) {
                    mbar_arrive_expect_tx(ffull + q, fb);
                    bulk_copy_g2s(fslots + q * fb, fsrc + (size_t)(st_lo + q) * fb, fb, ffull + q);
                }
            }
            issued = upto;
        };
        int slot = 0, round = 0;          // ring position, completed passes over the ring
        int eb = eb_first, eb_left = 0;   // current k-block, stages left in it
        for (int ks = 0; ks < nst; ++ks) {
            const int s = st_lo + ks;
            if (eb_left == 0) {
                // stage the k-block's scales (all 32 lanes), one block ahead of the consumers
                if (ks > 0) ++eb;
                eb_left = min(a.ebs * (eb + 1), st_hi) - s;
                const int ebl = eb - eb_first, b = ebl & 1;
                if (ebl >= 2) {
                    // the consumers release this buffer only after the digits of the
                    // stages before this one have reached them
                    if constexpr (!INK) issue_primed(min(ks, primed));
                    if (!timed_out) timed_out = !mbar_wait(sempty + b, (uint32_t)(((ebl >> 1) - 1) & 1));
                }
                int gA, ng;
                eb_groups(eb, gA, ng);
                // asynchronous copies: the producer never waits for them; rows past N copy
                // the last row's scales (their outputs are never stored). With rows of a
                // multiple of 4 scales, whole aligned 16-byte chunks around [gA, gA + ng) are
                // copied (a row keeps gA's offset inside its chunk, at most 12 floats).
                float *dst = scl + b * kRowsPerCta * kSG;
                if (vec16) {
                    const int c0 = gA & ~3, nc = (gA + ng + 3 - c0) >> 2;
                    for (int r = lane; r < kRowsPerCta; r += 32) {
                        const int n = min(cl * kRowsPerCta + r, a.N - 1);
                        const float *src = a.scales + (size_t)n * a.scales_per_row + c0;
                        for (int q = 0; q < nc; ++q) cp_async16(dst + r * kSG + 4 * q, src + 4 * q);
                    }
                } else {
                    for (int r = lane; r < kRowsPerCta; r += 32) {
                        const int n = min(cl * kRowsPerCta + r, a.N - 1);
                        const float *src = a.scales + (size_t)n * a.scales_per_row + gA;
                        for (int gi = 0; gi < ng; ++gi) cp_async4(dst + r * kSG + gi, src + gi);
                    }
                }
                cp_async_arrive(sfull + b);
            }
            --eb_left;
            if (round > 0 && !timed_out) timed_out = !mbar_wait(empty + slot, (uint32_t)((round - 1) & 1));
            if (lane == 0 && !timed_out) {
                mbar_arrive_expect_tx(full + slot, kPayloadBytes);
                tma_load_2d(slots + slot * kPayloadBytes, &tmap, full + slot, s * kTileBytes, cl * kRowsPerCta);
            }
            if constexpr (!INK) {
                const uint32_t fb = (uint32_t)a.fslot_bytes;
                if (ks >= primed) {
                    if (!timed_out) timed_out = !mbar_wait(fempty + slot, (uint32_t)((round - 1) & 1));
                    if (lane == 0 && !timed_out) {
                        mbar_arrive_expect_tx(ffull + slot, fb);
                        bulk_copy_g2s(fslots + slot * fb, fsrc + (size_t)s * fb, fb, ffull + slot);
                    }
                }
                if (ks == primed - 1) issue_primed(primed);  // the ring is primed with codes
            }
            if (++slot == nring) { slot = 0; ++round; }
        }
    } else {
        // ---------------- consumers ----------------
        const int g = lane >> 2, t = lane & 3;
        const int ct = threadIdx.x;  // 0..255
        if constexpr (INK) {
            // digits of this CTA's K range of the single activation row, built while the
            // first payload tiles are in flight; x may be the output of the kernel before
            // this one (a no-op unless this grid was launched as a dependent)
            grid_dep_wait();
            const int k_lo = st_lo * STAGEK, k_hi = min(st_hi * STAGEK, a.K);
            const int nu = max(k_hi - k_lo, 0) / 8;
            constexpr int R = kFragCap / 4 / 8 / kConsumerThreads;  // units per thread (4)
            float v[R][8];
#pragma unroll
            for (int r = 0; r < R; ++r) {
                const int u = ct + kConsumerThreads * r;
                if (u < nu) {
                    load_x8<XBF16>(a.x, (int64_t)k_lo + 8 * u, v[r]);
                } else {
#pragma unroll
                    for (int q = 0; q < 8; ++q) v[r][q] = 0.f;
                }
            }
#pragma unroll
            for (int r = 0; r < R; ++r) {
                // a warp's 32 units are 256 consecutive k: at most two k-blocks
                const int u = ct + kConsumerThreads * r;
                const int lb = u < nu ? (st_lo + (8 * u) / STAGEK) / a.ebs - eb_first : -1;
                const uint32_t m = absmax8(v[r]);
                const int lbA = __shfl_sync(0xffffffffu, lb, 0);
                const uint32_t mA = __reduce_max_sync(0xffffffffu, lb == lbA ? m : 0u);
                const uint32_t mB = __reduce_max_sync(0xffffffffu, (lb >= 0 && lb != lbA) ? m : 0u);
                if (lane == 0 && lbA >= 0) {
                    atomicMax(mx_sh + lbA, mA);
                    if (mB) atomicMax(mx_sh + lbA + 1, mB);
                }
            }
            named_barrier_sync(1, kConsumerThreads);
            uint2 *fbase = reinterpret_cast<uint2 *>(fslots);
#pragma unroll
            for (int r = 0; r < R; ++r) {
                const int u = ct + kConsumerThreads * r;
                if (u < nu) {
                    const int ls = (8 * u) / STAGEK;  // local stage
                    const int lb = (st_lo + ls) / a.ebs - eb_first;
                    const int sh = 30 - block_exp(mx_sh[lb]);
                    const int e1 = min(max(sh, -126), 127);
                    const float f1 = pow2(e1), f2 = pow2(min(max(sh - e1, -126), 127));
                    frag_unit<BITS, L>(fbase + (size_t)ls * (a.fslot_bytes / 8), 8 * u - ls * STAGEK, 0, v[r], f1,
                                       f2, 1, LW, true);
                }
            }
            named_barrier_sync(1, kConsumerThreads);
        } else {
            grid_dep_wait();  // the exponents are read from global memory
        }
        const int pr = 16 * warp + row_perm<L>(g);  // physical row of MMA row g in the CTA
        const int row0 = cl * kRowsPerCta + pr, row1 = row0 + 8;
        const bool ok0 = row0 < a.N, ok1 = row1 < a.N;
        uint32_t aoff[SPS];
#pragma unroll
        for (int sl = 0; sl < SPS; ++sl) {
            const int off = sl * 4 * L + t * L;
            aoff[sl] = pr * kTileBytes + (((off >> 4) ^ (pr & 7)) << 4) + (off & 15);
        }
        const int fl = lane & (LW - 1);  // lanes past the stored width repeat lanes (their columns are unused)
        // fold exponent of this lane's columns: 2^(E-30), 2^-4 for the int4 factor 16,
        // 2^16 for the high digit pair (t even)
        const int fadj = -30 - (BITS == 4 ? 4 : 0) + ((t & 1) == 0 ? 16 : 0);
        int c[NB][4];
        float y0[NB], y1[NB], acc0[NB], acc1[NB];
        int fe[NB], enext[NB];
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) {
            c[nb][0] = c[nb][1] = c[nb][2] = c[nb][3] = 0;
            y0[nb] = y1[nb] = acc0[nb] = acc1[nb] = 0.f;
            fe[nb] = enext[nb] = 0;
        }
        auto load_exps = [&](int eb) {
#pragma unroll
            for (int nb = 0; nb < NB; ++nb) {
                const int ml = 2 * nb + (t >> 1);
                enext[nb] = ml < mcnt ? a.ebexp[(int64_t)(mc * 16 + ml) * a.n_eb + eb] : 0;
            }
        };
        if constexpr (!INK) {
            if (nst > 0) load_exps(eb_first);
        }
        int lg = (st_lo * SPS) / a.spg;                 // group of the next segment
        int crem = a.spg - (st_lo * SPS - lg * a.spg);  // segments left in that group
        int gA = 0, ng = 0, b = 0;
        const float *sb = scl;
        auto flush = [&](int q) {  // a group (or a stage) ends: scale its exact sums
            const float s0 = sb[pr * kSG + q], s1 = sb[(pr + 8) * kSG + q];
#pragma unroll
            for (int nb = 0; nb < NB; ++nb) {
                const int p0 = c[nb][0] * 256 + c[nb][1], p1 = c[nb][2] * 256 + c[nb][3];
                y0[nb] = fmaf(s0, __int2float_rn(p0), y0[nb]);
                y1[nb] = fmaf(s1, __int2float_rn(p1), y1[nb]);
                c[nb][0] = c[nb][1] = c[nb][2] = c[nb][3] = 0;
            }
        };
        auto fold = [&]() {  // end of a k-block: apply its power of two exactly
#pragma unroll
            for (int nb = 0; nb < NB; ++nb) {
                acc0[nb] += scale2(y0[nb], fe[nb]);
                acc1[nb] += scale2(y1[nb], fe[nb]);
                y0[nb] = y1[nb] = 0.f;
            }
        };
        int slot = 0, round = 0;
        int eb = eb_first, eb_left = 0;
        for (int ks = 0; ks < nst; ++ks) {
            const int s = st_lo + ks;
            if (eb_left == 0) {
                if (ks > 0) {
                    fold();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(sempty + b);
                    ++eb;
                }
                eb_left = min(a.ebs * (eb + 1), st_hi) - s;
                const int ebl = eb - eb_first;
                b = ebl & 1;
                eb_groups(eb, gA, ng);
                sb = scl + b * kRowsPerCta * kSG + (vec16 ? (gA & 3) : 0);
                if constexpr (INK) {
                    fe[0] = block_exp(mx_sh[ebl]) + fadj;
                } else {
#pragma unroll
                    for (int nb = 0; nb < NB; ++nb) fe[nb] = enext[nb] + fadj;
                    if ((eb + 1) * a.ebs < st_hi) load_exps(eb + 1);  // one block ahead
                }
                if (!timed_out) timed_out = !mbar_wait(sfull + b, (uint32_t)((ebl >> 1) & 1));
            }
            --eb_left;
            const int nsl = min(SPS, seg_hi - s * SPS);  // valid segments (last stage may be short)
            if (!timed_out) timed_out = !mbar_wait(full + slot, (uint32_t)(round & 1));
            const uint8_t *stg = slots + slot * kPayloadBytes;
            uint32_t A0[SPS][WPT], A1[SPS][WPT];
#pragma unroll
            for (int sl = 0; sl < SPS; ++sl) {
                lds_words<L>(A0[sl], stg + aoff[sl]);
                lds_words<L>(A1[sl], stg + aoff[sl] + 8 * kTileBytes);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(empty + slot);  // the codes now live in registers: refill
            const uint8_t *fr;
            if constexpr (INK) {
                fr = fslots + ks * a.fslot_bytes;
            } else {
                if (!timed_out) timed_out = !mbar_wait(ffull + slot, (uint32_t)(round & 1));
                fr = fslots + slot * a.fslot_bytes;
            }
            if constexpr (GPS >= 0) {
                const int qb = (GPS > 0 ? s * GPS : (s * SPS) / a.spg) - gA;  // first group, in the k-block
                const float *s0p = sb + pr * kSG + qb, *s1p = s0p + 8 * kSG;
                const uint8_t *frl = fr + fl * (PAIRED ? 16 : 8);
                if (nsl == SPS)
                    stage_fixed<BITS, L, NB, LW, GPS, true>(A0, A1, frl, s0p, s1p, nsl, y0, y1);
                else
                    stage_fixed<BITS, L, NB, LW, GPS, false>(A0, A1, frl, s0p, s1p, nsl, y0, y1);
            } else {
                uint4 bq[PAIRED ? NB : 1];
#pragma unroll
                for (int i = 0; i < KTS; ++i) {
                    const int sl = i / KTI, j = i % KTI;
                    if (sl < nsl) {
                        uint32_t af[4];
                        unpack_a<BITS, L>(af, A0[sl], A1[sl], j);
#pragma unroll
                        for (int nb = 0; nb < NB; ++nb) {
                            uint32_t b0, b1;
                            if constexpr (PAIRED) {
                                if ((i & 1) == 0)
                                    bq[nb] = *reinterpret_cast<const uint4 *>(
                                        fr + 8 * (size_t)frag_idx(i, nb, fl, NB, LW, true));
                                b0 = (i & 1) ? bq[nb].z : bq[nb].x;
                                b1 = (i & 1) ? bq[nb].w : bq[nb].y;
                            } else {
                                const uint2 bb = *reinterpret_cast<const uint2 *>(
                                    fr + 8 * (size_t)frag_idx(i, nb, fl, NB, LW, false));
                                b0 = bb.x;
                                b1 = bb.y;
                            }
                            mma_s8_16832(c[nb], af, b0, b1);
                        }
                        if (j == KTI - 1) {  // end of a segment
                            const bool gend = --crem == 0;
                            if (gend || sl == nsl - 1) {
                                flush(lg - gA);
                                if (gend) {
                                    ++lg;
                                    crem = a.spg;
                                }
                            }
                        }
                    }
                }
            }
            if constexpr (!INK) {
                __syncwarp();
                if (lane == 0) mbar_arrive(fempty + slot);
            }
            if (++slot == nring) { slot = 0; ++round; }
        }
        if (nst > 0) fold();
        // high + low digit halves: lane t (even) takes lane t + 1's half
        float tot0[NB], tot1[NB];
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) {
            tot0[nb] = acc0[nb] + __shfl_xor_sync(0xffffffffu, acc0[nb], 1);
            tot1[nb] = acc1[nb] + __shfl_xor_sync(0xffffffffu, acc1[nb], 1);
        }
        if (a.CS == 1) {
            if ((t & 1) == 0) {
#pragma unroll
                for (int nb = 0; nb < NB; ++nb) {
                    const int ml = 2 * nb + (t >> 1);
                    if (ml < mcnt) {
                        float *yr = a.y + (int64_t)(mc * 16 + ml) * a.N;
                        if (ok0) yr[row0] = tot0[nb];
                        if (ok1) yr[row1] = tot1[nb];
                    }
                }
            }
        } else {
            named_barrier_sync(1, kConsumerThreads);  // every warp is done with the ring
            if ((t & 1) == 0) {
#pragma unroll
                for (int nb = 0; nb < NB; ++nb) {
                    const int ml = 2 * nb + (t >> 1);
                    if (ml < mcnt) {
                        red[pr * 16 + ml] = tot0[nb];
                        red[(pr + 8) * 16 + ml] = tot1[nb];
                    }
                }
            }
        }
    }
    if (timed_out && a.status) atomicOr(a.status, Q4_STATUS_TIMEOUT);
    if (a.CS == 1) return;

    // ---------------- cluster reduction of the K-split partial sums ----------------
    cluster_sync();
    const int rows_per = (kRowsPerCta + a.CS - 1) / a.CS;
    const int items = rows_per * mcnt;
    for (int it = threadIdx.x; it < items; it += kThreads) {
        const int rl = crank * rows_per + it / mcnt;  // row within the cluster's 128
        if (rl >= kRowsPerCta) break;
        const int ml = it % mcnt;
        const int n = cl * kRowsPerCta + rl;
        const float *src = red + rl * 16 + ml;  // same offset in every CTA of the cluster
        float pv[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) pv[q] = q < a.CS ? ld_dsmem_f32(src, (uint32_t)q) : 0.f;
        float sum = pv[0];
#pragma unroll
        for (int q = 1; q < 8; ++q) sum += pv[q];  // rank order; absent ranks add +0
        if (n < a.N) a.y[(int64_t)(mc * 16 + ml) * a.N + n] = sum;
    }
    cluster_sync();  // keep this CTA's shared memory alive until every peer has read it
}

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            p = nullptr;
        return reinterpret_cast<EncodeTiledFn>(p);
    }();
    return fn;
}

// early: the weights are static, so the call's first grid may start (and the stream
// kernel read payload and scales) while the previous kernel on the stream still runs.
// Every read of x, and every write, still waits for that kernel to finish.
template <int BITS, int L, int NB, int GPS, bool INK, bool XBF16>
cudaError_t launch_typed(const GemvPlan &pl, const GemvArgs &a, const CUtensorMap &tm, bool x_bf16,
                         bool early, cudaStream_t st) {
    cudaError_t err;
    cudaLaunchAttribute pdl;
    pdl.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl.val.programmaticStreamSerializationAllowed = 1;
    // chunks of 9-16 rows of x (NB == 8) ignore the flag: their early start was measured
    // slower (a Llama-7B-shaped decode step at M = 16: 4.93 ms against 4.81 ms)
    if (NB > 4) early = false;
    if constexpr (!INK) {
        cudaLaunchConfig_t pc = {};
        pc.gridDim = dim3(pl.n_eb, pl.nmc);
        pc.blockDim = dim3(256);
        pc.stream = st;
        pc.attrs = &pdl;
        pc.numAttrs = early ? 1 : 0;
        err = x_bf16 ? cudaLaunchKernelEx(&pc, gemv_prep<BITS, L, true>, a)
                     : cudaLaunchKernelEx(&pc, gemv_prep<BITS, L, false>, a);
        if (err != cudaSuccess) return err;
    }
    auto kern = gemv_stream<BITS, L, NB, GPS, INK, XBF16>;
    const size_t smem = pl.smem_bytes;
    err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(pl.clusters * pl.CS, pl.nmc);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = pl.CS;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1] = pdl;
    cfg.attrs = attr;
    // after gemv_prep the stream kernel always starts early (the prep grid itself began
    // only once everything before it had finished, unless the weights are static); the
    // one-kernel path starts early only with static weights
    cfg.numAttrs = INK && !early ? 1 : 2;
    return cudaLaunchKernelEx(&cfg, kern, a, tm);
}

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

cudaError_t dispatch_gemv(const GemvPlan &pl, const GemvArgs &a, const CUtensorMap &tm, bool x_bf16,
                          bool early, cudaStream_t st) {
#define Q4_INK(B, LL, G)                                                                         \
    if (pl.bits == B && pl.L == LL && pl.gps == G)                                               \
        return x_bf16 ? launch_typed<B, LL, 1, G, true, true>(pl, a, tm, true, early, st)        \
                      : launch_typed<B, LL, 1, G, true, false>(pl, a, tm, false, early, st);
#define Q4_STAGED(B, LL, G)                                                                      \
    if (pl.bits == B && pl.L == LL && pl.gps == G) {                                             \
        switch (pl.NB) {                                                                         \
            case 1: return launch_typed<B, LL, 1, G, false, false>(pl, a, tm, x_bf16, early, st); \
            case 2: return launch_typed<B, LL, 2, G, false, false>(pl, a, tm, x_bf16, early, st); \
            case 4: return launch_typed<B, LL, 4, G, false, false>(pl, a, tm, x_bf16, early, st); \
            default: return launch_typed<B, LL, 8, G, false, false>(pl, a, tm, x_bf16, early, st); \
        }                                                                                        \
    }
#define Q4_ALL(M)                                                                                \
    M(4, 16, 2) M(4, 16, 0) M(4, 8, 4) M(4, 4, 8) M(4, 4, -1) M(8, 16, 2) M(8, 16, 0) M(8, 8, 4) M(8, 8, -1)
    if (pl.ink) {
        Q4_ALL(Q4_INK)
    } else {
        Q4_ALL(Q4_STAGED)
    }
#undef Q4_ALL
#undef Q4_STAGED
#undef Q4_INK
    return cudaErrorInvalidValue;
}

}  // namespace

bool gemv_plan(int64_t M, int64_t N, int64_t K, int bits, int64_t group, int sms, GemvPlan *pl) {
    GemvPlan p = {};
    p.bits = bits;
    if (K % 32 != 0 || group <= 0 || K % group != 0) return false;
    // a segment (4 lanes x L bytes of a row) must lie inside one scale group
    if (bits == 4)
        p.L = group % 128 == 0 ? 16 : group % 64 == 0 ? 8 : group % 32 == 0 ? 4 : 0;
    else
        p.L = group % 64 == 0 ? 16 : group % 32 == 0 ? 8 : 0;
    if (!p.L) return false;
    // groups per 128-byte stage when they divide it, 0 when the stage lies inside one
    // group, -1 otherwise (then the narrowest segments, which always fit in a group)
    {
        const int64_t sk = kTileBytes * 8 / bits;
        p.gps = sk % group == 0 ? (int)(sk / group) : group % sk == 0 ? 0 : -1;
        if (p.gps == 1) p.gps = 0;  // one group per stage: the same as a stage inside a group
        if (p.gps < 0) p.L = bits == 4 ? 4 : 8;
    }
    if (K > ((int64_t)1 << 30) || N > ((int64_t)1 << 30) || M > (int64_t)65535 * 16) return false;
    p.segk = 32 * p.L / bits;
    p.segs = (int)(K / p.segk);
    p.spg = (int)(group / p.segk);
    p.nmc = (int)((M + 15) / 16);
    const int mc0 = (int)(M < 16 ? M : 16);
    const int nbm = (mc0 + 1) / 2;  // n8 blocks needed: two rows of x (4 digits each) per block
    p.NB = nbm <= 1 ? 1 : nbm <= 2 ? 2 : nbm <= 4 ? 4 : 8;
    p.paired = p.NB <= 2;
    p.clusters = (int)((N + kRowsPerCta - 1) / kRowsPerCta);
    const int64_t rowbytes = K * bits / 8;
    p.stages_total = (int)((rowbytes + kTileBytes - 1) / kTileBytes);
    const int stagek = kTileBytes * 8 / bits;
    // k-block: about kGroupsPerBlock scale groups and at most kBlockK k, in whole stages
    int64_t ebs = kGroupsPerBlock * group / stagek;
    if (ebs > kBlockK / stagek) ebs = kBlockK / stagek;
    if (ebs < 1) ebs = 1;
    p.ebs = (int)ebs;
    p.n_eb = (p.stages_total + p.ebs - 1) / p.ebs;
    // split K over a cluster so that the grid is one wave of two CTAs per SM
    const int64_t slots = (int64_t)sms * 2;
    const int64_t blocks = (int64_t)p.clusters * p.nmc;
    int64_t cs = slots / (blocks > 0 ? blocks : 1);
    if (cs > 8) cs = 8;
    if (cs > p.stages_total / 2) cs = p.stages_total / 2;
    p.CS = cs < 1 ? 1 : (int)cs;
    p.stages_per_cta = (p.stages_total + p.CS - 1) / p.CS;
    const int kts = bits == 4 ? 8 : 4;  // MMAs per stage
    // one row of x: 16 digit lanes, built on chip when the CTA's K range fits
    p.ink = M == 1 && (int64_t)p.stages_per_cta * kts * 16 * 8 <= kFragCap;
    p.lw = p.ink ? 16 : 32;
    p.fslot_bytes = kts * p.NB * p.lw * 8;
    const size_t fixed = 1024 + 2 * (size_t)kRowsPerCta * kSG * 4 + kMaxLocalBlocks * 4 + (4 * kMaxStages + 4) * 8;
    int nr;
    if (p.ink) {
        const size_t frag = (size_t)p.stages_per_cta * p.fslot_bytes;
        nr = (int)((kSmemBudget - fixed - frag) / kPayloadBytes);
        p.nst_ring = nr > kMaxStages ? kMaxStages : nr < 2 ? 2 : nr;
        p.smem_bytes = fixed + frag + (size_t)p.nst_ring * kPayloadBytes;
    } else {
        nr = (int)((kSmemBudget - fixed) / (kPayloadBytes + p.fslot_bytes));
        p.nst_ring = nr > kMaxStages ? kMaxStages : nr < 2 ? 2 : nr;
        p.smem_bytes = fixed + (size_t)p.nst_ring * (kPayloadBytes + p.fslot_bytes);
    }
    static_assert(kRedBytes <= 2 * kPayloadBytes, "partial sums fit in the ring");
    // workspace (several rows of x): digits [mc][stage][fslot_bytes], then exponents [mc*16][n_eb]
    if (p.ink) {
        p.off_frag = p.off_exp = p.bytes = 0;
    } else {
        p.off_frag = 0;
        p.off_exp = align_up((size_t)p.nmc * p.stages_total * p.fslot_bytes, 256);
        p.bytes = align_up(p.off_exp + (size_t)p.nmc * 16 * p.n_eb * 4, 256);
    }
    *pl = p;
    return true;
}

cudaError_t launch_gemv(const GemvPlan &pl, const void *x, bool x_bf16, int64_t M,
                        const uint8_t *payload, const float *scales, int64_t N, int64_t K,
                        int64_t group, float *y, void *ws, uint32_t *status, bool weights_static,
                        cudaStream_t st) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return cudaErrorNotSupported;
    const uint64_t rowbytes = (uint64_t)K * pl.bits / 8;
    CUtensorMap tm;
    const cuuint64_t dims[2] = {rowbytes, (cuuint64_t)N};
    const cuuint64_t strides[1] = {rowbytes};
    const cuuint32_t box[2] = {(cuuint32_t)kTileBytes, (cuuint32_t)kRowsPerCta};
    const cuuint32_t estr[2] = {1, 1};
    if (enc(&tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(payload), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    char *w = static_cast<char *>(ws);
    GemvArgs a;
    a.scales = scales;
    a.x = x;
    a.y = y;
    a.status = status;
    a.frag = w ? reinterpret_cast<uint8_t *>(w + pl.off_frag) : nullptr;
    a.ebexp = w ? reinterpret_cast<int *>(w + pl.off_exp) : nullptr;
    a.M = (int)M;
    a.N = (int)N;
    a.K = (int)K;
    a.segs = pl.segs;
    a.spg = pl.spg;
    a.scales_per_row = (int)(K / group);
    a.CS = pl.CS;
    a.stages_total = pl.stages_total;
    a.stages_per_cta = pl.stages_per_cta;
    a.ebs = pl.ebs;
    a.n_eb = pl.n_eb;
    a.lw = pl.lw;
    a.NB = pl.NB;
    a.paired = pl.paired;
    a.nst_ring = pl.nst_ring;
    a.fslot_bytes = pl.fslot_bytes;
    return dispatch_gemv(pl, a, tm, x_bf16, weights_static, st);
}

}  // namespace q4
