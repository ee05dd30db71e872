// gemv.cu -- fused unpack -> dequant -> GEMV for decode (x in chunks of 16 rows).
//
// y[m][n] = sum_k x[m][k] * w'[n][k], w' = code * scale (pack()/unpack() of the
// "量化推理" page; the QuantizedMatmul of "Huit bits, puis quatre", which reads the
// codes in generation products, where one waits on memory). The packed weights are the
// whole cost, so the kernel is built around streaming them:
//
//   gemv_prep   (tiny grid) turns x into tensor-core B fragments once per call: every
//               activation row m is split exactly into x' = hi + lo (two fp16 values,
//               22 significant bits) after a power-of-two rescale x' = x * 2^-e whose e is
//               chosen per (m, block of k) so that the block maximum lands in
//               [2^14, 2^15); the fragments go to a global workspace in the exact order
//               the MMA wants them, the exponents next to them.
//   gemv_stream (one wave: up to two CTAs per SM) streams the codes. A producer warp
//               issues, per stage, one 2D TMA load of a 128-row x 128-byte tile of the
//               payload (128-byte swizzle) plus one bulk copy of the matching fragment
//               tile into a 4-deep shared-memory ring guarded by full/empty mbarriers,
//               and loads each k-block's scales into double-buffered shared memory one
//               block ahead. Eight consumer warps decode and multiply; they do no
//               staging work of their own. It is launched as a programmatic dependent
//               of gemv_prep: the payload loads start before the fragments exist, and
//               only the fragment copies wait (griddepcontrol.wait).
//
// Tensor cores (warp-level mma.sync m16n8k16, fp16 operands, fp32 accumulation):
//   A = 16 weight rows x 16 k of CODES, exact in fp16 (|code| <= 127).
//   B = 16 k x 8 columns: columns 2c and 2c+1 hold hi and lo of one activation row,
//       so one lane owns both partial sums of the same (weight row, m) in c0/c1.
//   When a scale group ends, the lane multiplies the partial sum by the group's fp32
//   scale and adds it to an fp32 accumulator; no arithmetic on w' is done in fp16. At
//   the end of each k-block the block's 2^e is applied exactly.
// Inside a group the order of k is permuted so that a lane builds its A fragment from
// one shared-memory read; the fragments use the same permutation. Rows are permuted
// inside each 16-row tile so those reads are free of bank conflicts.
//
// A thread-block cluster of CS CTAs splits K; the CS partial sums meet in distributed
// shared memory (fixed rank order), so results do not depend on timing. Every wait is
// bounded; one that gives up sets Q4_STATUS_TIMEOUT in the optional status word.
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
constexpr int kSG = 17;                            // scale slots per row per k-block (odd)

struct GemvArgs {
    const float *scales;
    const void *x;
    float *y;
    uint32_t *status;
    const uint8_t *frag;  // global fragments: [mc][k-tile][nb][LW lanes] x uint2
    int *ebexp;           // exponents: [mc*16 + m][n_eb]
    int M, N, K;
    int segs, spg, scales_per_row;
    int CS;               // CTAs per cluster = K splits
    int stages_total;     // 128-byte tiles per weight row (last may be partial)
    int stages_per_cta;
    int ebs;              // stages per k-block (exponent + scale block)
    int n_eb;
    int lw;               // fragment lanes stored per (k-tile, nb): 8*M for one block of <= 4 rows, else 32
    int nst_ring;         // stages in the ring (<= kMaxStages)
    int slot_bytes;       // payload + fragment bytes of one ring slot (1024-aligned)
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

template <bool XBF16>
Q4_DEVINL void load_x4(const void *x, int64_t idx, float (&v)[4]) {
    if constexpr (XBF16) {
        const uint2 b = *reinterpret_cast<const uint2 *>(reinterpret_cast<const uint16_t *>(x) + idx);
        v[0] = __uint_as_float(b.x << 16);
        v[1] = __uint_as_float(b.x & 0xffff0000u);
        v[2] = __uint_as_float(b.y << 16);
        v[3] = __uint_as_float(b.y & 0xffff0000u);
    } else {
        const float4 f = *reinterpret_cast<const float4 *>(reinterpret_cast<const float *>(x) + idx);
        v[0] = f.x; v[1] = f.y; v[2] = f.z; v[3] = f.w;
    }
}

// Exact split of a pair of rescaled activations into fp16 (hi, lo) pairs.
Q4_DEVINL void split2(float a, float b, uint32_t &hi, uint32_t &lo) {
    const __half2 h = __floats2half2_rn(a, b);
    const float2 hf = __half22float2(h);
    const __half2 l = __floats2half2_rn(a - hf.x, b - hf.y);  // a - hf.x is exact (Sterbenz)
    hi = *reinterpret_cast<const uint32_t *>(&h);
    lo = *reinterpret_cast<const uint32_t *>(&l);
}
Q4_DEVINL uint32_t pack_lo_halves(uint32_t p, uint32_t q) { return prmt(p, q, 0x5410u); }  // (p.x, q.x)
Q4_DEVINL uint32_t pack_hi_halves(uint32_t p, uint32_t q) { return prmt(p, q, 0x7632u); }  // (p.y, q.y)
Q4_DEVINL float pow2(int e) { return __int_as_float((e + 127) << 23); }  // 2^e, e in [-126, 127]

// One CTA per (k-block eb, 16-row chunk mc of x): exponent per activation row, then the
// B fragments of the block in MMA order. It lets the dependent stream kernel start at once.
template <int BITS, int L, int NB, bool XBF16>
__global__ void __launch_bounds__(256) gemv_prep(const GemvArgs a) {
    grid_dep_launch();
    constexpr int SEGK = 32 * L / BITS;
    constexpr int KT = SEGK / 16;
    constexpr int STAGEK = kTileBytes * 8 / BITS;
    constexpr int BLK = BITS == 4 ? 8 : 4;  // k per work item
    __shared__ uint32_t mx_sh[16];
    __shared__ int e_sh[16];
    const int eb = blockIdx.x, mc = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int mcnt = min(16, a.M - mc * 16);
    const int k0 = eb * a.ebs * STAGEK;
    const int k1 = min(a.K, k0 + a.ebs * STAGEK);
    const int nk = k1 - k0;
    // (a) exponent per activation row
    for (int ml = warp; ml < 16; ml += 8) {
        uint32_t mx = 0;
        if (ml < mcnt) {
            const int64_t rowb = (int64_t)(mc * 16 + ml) * a.K + k0;
            // a k-block is at most 2048 values: 16 loads per lane, all in flight at once
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int k = lane * 4 + 128 * i;
                if (k < nk) {
                    float v[4];
                    load_x4<XBF16>(a.x, rowb + k, v);
#pragma unroll
                    for (int q = 0; q < 4; ++q) mx = max(mx, __float_as_uint(v[q]) & 0x7fffffffu);
                }
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        if (lane == 0) {
            int e = 0;
            if (mx != 0 && mx < 0x7f800000u) {
                int E;
                frexpf(__uint_as_float(mx), &E);  // max|x| in [2^(E-1), 2^E)
                e = E - 15;                        // -> max|x| * 2^-e in [2^14, 2^15)
            }
            e_sh[ml] = e;
            a.ebexp[(int64_t)(mc * 16 + ml) * a.n_eb + eb] = e;
        }
    }
    __syncthreads();
    // (b) fragments of absent activation rows are zero (only the 32-lane layout has any)
    const int64_t kt0 = k0 / 16, nkt = nk / 16;
    uint2 *frag = reinterpret_cast<uint2 *>(const_cast<uint8_t *>(a.frag)) +
                  ((int64_t)mc * (a.K / 16) + kt0) * NB * a.lw;
    if (a.lw == 32 && mcnt < 4 * NB) {
        for (int64_t i = threadIdx.x; i < nkt * NB * 32; i += blockDim.x) {
            const int ln = (int)(i & 31), nb = (int)((i >> 5) % NB);
            if (nb * 4 + (ln >> 3) >= mcnt) frag[i] = make_uint2(0u, 0u);
        }
    }
    // (c) rescale, split, scatter into fragment order
    const int nblk = nk / BLK;
    for (int it = threadIdx.x; it < nblk * mcnt; it += blockDim.x) {
        const int ml = it / nblk, blk = it - ml * nblk;
        const int e = e_sh[ml];
        // x * 2^-e as two exact power-of-two multiplications (2^-e may leave fp32 range)
        const int e1 = min(max(-e, -126), 127);
        const float f1 = pow2(e1), f2 = pow2(min(max(-e - e1, -126), 127));
        const int64_t xb = (int64_t)(mc * 16 + ml) * a.K + k0 + blk * BLK;
        float v[8];
        {
            float t4[4];
            load_x4<XBF16>(a.x, xb, t4);
#pragma unroll
            for (int q = 0; q < 4; ++q) v[q] = (t4[q] * f1) * f2;
            if constexpr (BLK == 8) {
                load_x4<XBF16>(a.x, xb + 4, t4);
#pragma unroll
                for (int q = 0; q < 4; ++q) v[4 + q] = (t4[q] * f1) * f2;
            }
        }
        const int kl = blk * BLK;  // k offset inside the block (blocks start on segment bounds)
        const int sl = kl / SEGK, within = kl - sl * SEGK;
        const int nb = ml >> 2, lane_hi = 8 * (ml & 3);
        if constexpr (BITS == 4) {
            // the 8 values are word w of lane quad t: k-tile 2w takes k {0,4 | 1,5},
            // k-tile 2w+1 takes k {2,6 | 3,7}
            const int t = within / (2 * L), w = (within % (2 * L)) / 8;
            uint32_t h01, l01, h45, l45, h23, l23, h67, l67;
            split2(v[0], v[1], h01, l01);
            split2(v[4], v[5], h45, l45);
            split2(v[2], v[3], h23, l23);
            split2(v[6], v[7], h67, l67);
            uint2 *f0 = frag + ((int64_t)(sl * KT + 2 * w) * NB + nb) * a.lw + lane_hi + t;
            uint2 *f1p = f0 + NB * a.lw;  // next k-tile
            f0[0] = make_uint2(pack_lo_halves(h01, h45), pack_hi_halves(h01, h45));
            f0[4] = make_uint2(pack_lo_halves(l01, l45), pack_hi_halves(l01, l45));
            f1p[0] = make_uint2(pack_lo_halves(h23, h67), pack_hi_halves(h23, h67));
            f1p[4] = make_uint2(pack_lo_halves(l23, l67), pack_hi_halves(l23, l67));
        } else {
            // the 4 values are word j of lane quad t, in natural order
            const int t = within / L, j = (within % L) / 4;
            uint32_t h01, l01, h23, l23;
            split2(v[0], v[1], h01, l01);
            split2(v[2], v[3], h23, l23);
            uint2 *f0 = frag + ((int64_t)(sl * KT + j) * NB + nb) * a.lw + lane_hi + t;
            f0[0] = make_uint2(h01, h23);
            f0[4] = make_uint2(l01, l23);
        }
    }
}

// ---- decode of the packed codes ------------------------------------------------------
// A fragment of k-tile j from one lane's words of row g (w0) and row g+8 (w1).
template <int BITS, int L>
Q4_DEVINL void unpack_a(uint32_t (&a)[4], const uint32_t (&w0)[L / 4], const uint32_t (&w1)[L / 4],
                        int j) {
    if constexpr (BITS == 4) {
        // fp16 0x6400 | u = 1024 + u; (1024 + u) - 1032 = u - 8 = code (exact)
        // fp16 0x6400 | (u << 4) = 1024 + 16u; (1024 + 16u) / 16 - 72 = code (exact)
        const uint32_t kMagic = 0x64006400u, kSub = 0x64086408u /* 1032 */;
        const uint32_t kInv16 = 0x2c002c00u /* 1/16 */, kNeg72 = 0xd480d480u /* -72 */;
        uint32_t x0 = w0[j >> 1], x1 = w1[j >> 1];
        if (j & 1) { x0 >>= 8; x1 >>= 8; }
        a[0] = hsub2(and_or(x0, 0x000f000fu, kMagic), kSub);
        a[1] = hsub2(and_or(x1, 0x000f000fu, kMagic), kSub);
        a[2] = hfma2(and_or(x0, 0x00f000f0u, kMagic), kInv16, kNeg72);
        a[3] = hfma2(and_or(x1, 0x00f000f0u, kMagic), kInv16, kNeg72);
    } else {
        // bytes biased by 128 then placed under exponent 0x64: 1024 + (code + 128); minus 1152
        const uint32_t kHi = 0x64646464u, kSub = 0x64806480u /* 1152 */;
        const uint32_t x0 = w0[j] ^ 0x80808080u, x1 = w1[j] ^ 0x80808080u;
        a[0] = hsub2(prmt(x0, kHi, 0x5140u), kSub);
        a[1] = hsub2(prmt(x1, kHi, 0x5140u), kSub);
        a[2] = hsub2(prmt(x0, kHi, 0x7362u), kSub);
        a[3] = hsub2(prmt(x1, kHi, 0x7362u), kSub);
    }
}


// Physical row (0..7) inside a 16-row tile of logical MMA row g (and g + 8), chosen so
// that the shared-memory reads of one instruction hit distinct banks under the
// 128-byte swizzle (8 lanes per phase for 16-byte reads, 16 for 8-byte, 32 for 4-byte).
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

// One segment: KT k-tiles of MMAs. Z: the accumulators start from zero (first k-tiles use
// a zero C operand instead of clearing registers).
template <int BITS, int L, int NB, int LW, int ACC, bool Z>
Q4_DEVINL void seg_mma(float (&c)[ACC][NB][4], const uint32_t (&w0)[L / 4], const uint32_t (&w1)[L / 4],
                       const uint2 *fk, bool stored) {
    constexpr int KT = (32 * L / BITS) / 16;
#pragma unroll
    for (int j = 0; j < KT; ++j) {
        uint32_t af[4];
        unpack_a<BITS, L>(af, w0, w1, j);
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) {
            const uint2 bb = fk[stored ? j * NB * LW + nb * LW : 0];
            if (Z && j < ACC)
                mma_f16_16816_z(c[j % ACC][nb], af, bb.x, bb.y);
            else
                mma_f16_16816(c[j % ACC][nb], af, bb.x, bb.y);
        }
    }
}

// One stage whose GPS scale groups each lie inside it: per-group accumulator chains
// (two alternating chains when GPS == 1), each started with a zero-C MMA, then every
// group is flushed with its scale. FULL: all SPS segments are valid (no branches).
template <int BITS, int L, int NB, int LW, int GPS, bool FULL>
Q4_DEVINL void stage_groups(const uint32_t (&A0)[kTileBytes / (4 * L)][L / 4],
                            const uint32_t (&A1)[kTileBytes / (4 * L)][L / 4], const uint2 *fr, bool stored,
                            const float *sb, int pr, int g0, int nsl, float (&pa0)[NB], float (&pa1)[NB]) {
    constexpr int KT = (32 * L / BITS) / 16;
    constexpr int SPS = kTileBytes / (4 * L);
    constexpr int SPG = SPS / GPS;  // segments per group
    constexpr int CH = GPS >= 2 ? GPS : 2;
    float cc[CH][NB][4];
#pragma unroll
    for (int sl = 0; sl < SPS; ++sl) {
        if (FULL || sl < nsl) {
#pragma unroll
            for (int j = 0; j < KT; ++j) {
                uint32_t af[4];
                unpack_a<BITS, L>(af, A0[sl], A1[sl], j);
                const int q = GPS >= 2 ? sl / SPG : ((sl * KT + j) & 1);
                const bool first = GPS >= 2 ? (sl % SPG == 0 && j == 0) : (sl * KT + j < 2);
#pragma unroll
                for (int nb = 0; nb < NB; ++nb) {
                    const uint2 bb = fr[stored ? (sl * KT + j) * NB * LW + nb * LW : 0];
                    if (first)
                        mma_f16_16816_z(cc[q][nb], af, bb.x, bb.y);
                    else
                        mma_f16_16816(cc[q][nb], af, bb.x, bb.y);
                }
            }
        }
    }
#pragma unroll
    for (int q = 0; q < GPS; ++q) {
        if (FULL || q * SPG < nsl) {
            const float s0 = sb[pr * kSG + g0 + q], s1 = sb[(pr + 8) * kSG + g0 + q];
#pragma unroll
            for (int nb = 0; nb < NB; ++nb) {
                float h0 = cc[q][nb][0] + cc[q][nb][1], h1 = cc[q][nb][2] + cc[q][nb][3];
                if constexpr (GPS == 1) {
                    h0 += cc[1][nb][0] + cc[1][nb][1];
                    h1 += cc[1][nb][2] + cc[1][nb][3];
                }
                pa0[nb] = fmaf(s0, h0, pa0[nb]);
                pa1[nb] = fmaf(s1, h1, pa1[nb]);
            }
        }
    }
}

Q4_DEVINL void bulk_copy_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// GPS > 0: every scale group lies inside one stage and a stage holds GPS whole groups
// (the group size divides the 256-k / 128-k stage); GPS == 0: any group size that is a
// multiple of a segment, tracked segment by segment.
template <int BITS, int L, int NB, int LW, int GPS>
__global__ void __launch_bounds__(kThreads, 2)
gemv_stream(const GemvArgs a, const __grid_constant__ CUtensorMap tmap) {
    constexpr int SEGK = 32 * L / BITS;
    constexpr int KT = SEGK / 16;
    constexpr int WPT = L / 4;
    constexpr int SPS = kTileBytes / (4 * L);  // segments per stage
    constexpr int KTS = SPS * KT;              // k-tiles per stage
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const int nring = a.nst_ring;
    uint8_t *slots = smem;                                  // codes: nring x 16 KB (1024-aligned)
    uint8_t *fslots = smem + nring * kPayloadBytes;         // fragments: nring x slot_bytes
    float *scl = reinterpret_cast<float *>(fslots + nring * a.slot_bytes);  // [2][128][kSG]
    float *red = scl + 2 * kRowsPerCta * kSG;                               // [128][16] when CS > 1
    uint2 *zero8 = reinterpret_cast<uint2 *>(red + (a.CS > 1 ? kRowsPerCta * 16 : 0));
    uint64_t *full = reinterpret_cast<uint64_t *>(zero8 + 2);  // codes landed
    uint64_t *empty = full + kMaxStages;                         // codes copied to registers
    uint64_t *ffull = empty + kMaxStages;                        // fragments landed
    uint64_t *fempty = ffull + kMaxStages;                       // fragments no longer read
    uint64_t *sfull = fempty + kMaxStages;
    uint64_t *sempty = sfull + 2;

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
    constexpr int ktile_bytes = NB * LW * 8;  // fragment bytes of one k-tile

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
        zero8[0] = zero8[1] = make_uint2(0u, 0u);
        fence_barrier_init();
    }
    __syncthreads();

    // groups [gA, gA + ng) touched by k-block eb inside this CTA's range
    auto eb_groups = [&](int eb, int &gA, int &ng) {
        const int s0 = max(st_lo, eb * a.ebs), s1 = min(st_hi, (eb + 1) * a.ebs);
        const int sg0 = s0 * SPS, sg1 = min(s1 * SPS, a.segs);
        gA = sg0 / a.spg;
        ng = (sg1 - 1) / a.spg - gA + 1;
    };

    bool timed_out = false;
    if (warp == kConsumers) {
        // ---------------- producer warp ----------------
        const uint8_t *fsrc = a.frag + (size_t)mc * (a.K / 16) * ktile_bytes;
        const int primed = min(nst, nring);
        int slot = 0, round = 0;          // ring position, completed passes over the ring
        int eb = eb_first, eb_left = 0;   // current k-block, stages left in it
        for (int ks = 0; ks < nst; ++ks) {
            const int s = st_lo + ks;
            if (eb_left == 0) {
                // stage the k-block's scales (all 32 lanes), one block ahead of the consumers
                if (ks > 0) ++eb;
                eb_left = min(a.ebs * (eb + 1), st_hi) - s;
                const int ebl = eb - eb_first, b = ebl & 1;
                if (ebl >= 2 && !timed_out) timed_out = !mbar_wait(sempty + b, (uint32_t)(((ebl >> 1) - 1) & 1));
                int gA, ng;
                eb_groups(eb, gA, ng);
                // asynchronous 4-byte copies: the producer never waits for them; rows past
                // N copy the last row's scales (their outputs are never stored)
                float *dst = scl + b * kRowsPerCta * kSG;
                for (int r = lane; r < kRowsPerCta; r += 32) {
                    const int n = min(cl * kRowsPerCta + r, a.N - 1);
                    const float *src = a.scales + (size_t)n * a.scales_per_row + gA;
                    for (int gi = 0; gi < ng; ++gi) cp_async4(dst + r * kSG + gi, src + gi);
                }
                cp_async_arrive(sfull + b);
            }
            --eb_left;
            const int ktv = min(KTS, a.K / 16 - s * KTS);
            const uint32_t fbytes = (uint32_t)(ktv * ktile_bytes);
            if (round > 0 && !timed_out) timed_out = !mbar_wait(empty + slot, (uint32_t)((round - 1) & 1));
            if (lane == 0 && !timed_out) {
                mbar_arrive_expect_tx(full + slot, kPayloadBytes);
                tma_load_2d(slots + slot * kPayloadBytes, &tmap, full + slot, s * kTileBytes, cl * kRowsPerCta);
            }
            if (ks >= primed) {
                if (!timed_out) timed_out = !mbar_wait(fempty + slot, (uint32_t)((round - 1) & 1));
                if (lane == 0 && !timed_out) {
                    mbar_arrive_expect_tx(ffull + slot, fbytes);
                    bulk_copy_g2s(fslots + slot * a.slot_bytes, fsrc + (size_t)s * KTS * ktile_bytes, fbytes,
                                  ffull + slot);
                }
            }
            if (ks == primed - 1) {
                // the ring is primed with codes; the fragments come from gemv_prep
                grid_dep_wait();
                if (lane == 0 && !timed_out) {
                    for (int q = 0; q < primed; ++q) {
                        const int sq = st_lo + q;
                        const uint32_t fq = (uint32_t)(min(KTS, a.K / 16 - sq * KTS) * ktile_bytes);
                        mbar_arrive_expect_tx(ffull + q, fq);
                        bulk_copy_g2s(fslots + q * a.slot_bytes, fsrc + (size_t)sq * KTS * ktile_bytes, fq, ffull + q);
                    }
                }
            }
            if (++slot == nring) { slot = 0; ++round; }
        }
    } else {
        // ---------------- consumers ----------------
        grid_dep_wait();  // the exponents are read from global memory
        const int g = lane >> 2, t = lane & 3;
        const int pr = 16 * warp + row_perm<L>(g);  // physical row of MMA row g in the CTA
        const int row0 = cl * kRowsPerCta + pr, row1 = row0 + 8;
        const bool ok0 = row0 < a.N, ok1 = row1 < a.N;
        uint32_t aoff[SPS];
#pragma unroll
        for (int sl = 0; sl < SPS; ++sl) {
            const int off = sl * 4 * L + t * L;
            aoff[sl] = pr * kTileBytes + (((off >> 4) ^ (pr & 7)) << 4) + (off & 15);
        }
        const bool stored = lane < LW;  // lanes beyond the stored width read zeros
        constexpr int ACC = NB == 1 ? 2 : 1;  // two accumulator chains when there is one column block
        float acc0[NB], acc1[NB], pa0[NB], pa1[NB], c[ACC][NB][4];
        int ecur[NB];
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) {
            acc0[nb] = acc1[nb] = pa0[nb] = pa1[nb] = 0.f;
            ecur[nb] = 0;
#pragma unroll
            for (int q = 0; q < ACC; ++q) c[q][nb][0] = c[q][nb][1] = c[q][nb][2] = c[q][nb][3] = 0.f;
        }
        int lg = (st_lo * SPS) / a.spg;                 // group of the next segment
        int crem = a.spg - (st_lo * SPS - lg * a.spg);  // segments left in that group
        int gA = 0, ng = 0, b = 0;
        bool fresh = true;                              // the accumulators hold nothing yet
        const float *sb = scl;
        auto flush = [&]() {
            const float s0 = sb[pr * kSG + (lg - gA)], s1 = sb[(pr + 8) * kSG + (lg - gA)];
#pragma unroll
            for (int nb = 0; nb < NB; ++nb) {
                float h0 = c[0][nb][0] + c[0][nb][1], h1 = c[0][nb][2] + c[0][nb][3];
                if constexpr (ACC == 2) {
                    h0 += c[1][nb][0] + c[1][nb][1];
                    h1 += c[1][nb][2] + c[1][nb][3];
                }
                pa0[nb] = fmaf(s0, h0, pa0[nb]);
                pa1[nb] = fmaf(s1, h1, pa1[nb]);
#pragma unroll
                for (int q = 0; q < ACC; ++q) c[q][nb][0] = c[q][nb][1] = c[q][nb][2] = c[q][nb][3] = 0.f;
            }
            fresh = true;
        };
        auto fold = [&]() {  // end of a k-block: apply its 2^e exactly
#pragma unroll
            for (int nb = 0; nb < NB; ++nb) {
                acc0[nb] += ldexpf(pa0[nb], ecur[nb]);
                acc1[nb] += ldexpf(pa1[nb], ecur[nb]);
                pa0[nb] = pa1[nb] = 0.f;
            }
        };
        int slot = 0, round = 0;
        int eb = eb_first, eb_left = 0;
        for (int ks = 0; ks < nst; ++ks) {
            const int s = st_lo + ks;
            if (eb_left == 0) {
                if (ks > 0) {
                    if (!fresh) flush();  // a group cut by the k-block boundary
                    fold();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(sempty + b);
                    ++eb;
                }
                eb_left = min(a.ebs * (eb + 1), st_hi) - s;
                const int ebl = eb - eb_first;
                b = ebl & 1;
                eb_groups(eb, gA, ng);
                sb = scl + b * kRowsPerCta * kSG;
#pragma unroll
                for (int nb = 0; nb < NB; ++nb) {
                    const int ml = nb * 4 + t;
                    ecur[nb] = ml < mcnt ? a.ebexp[(int64_t)(mc * 16 + ml) * a.n_eb + eb] : 0;
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
            if (!timed_out) timed_out = !mbar_wait(ffull + slot, (uint32_t)(round & 1));
            const uint2 *fr = stored ? reinterpret_cast<const uint2 *>(fslots + slot * a.slot_bytes) + lane : zero8;
            if constexpr (GPS > 0) {
                // whole groups inside the stage: one accumulator chain per group (two
                // alternating chains when the stage is one group), all flushed at its end.
                // A full stage is one branch-free block, so the chains interleave.
                const int g0 = s * GPS - gA;  // this stage's first group, relative to the k-block
                if (nsl == SPS)
                    stage_groups<BITS, L, NB, LW, GPS, true>(A0, A1, fr, stored, sb, pr, g0, SPS, pa0, pa1);
                else
                    stage_groups<BITS, L, NB, LW, GPS, false>(A0, A1, fr, stored, sb, pr, g0, nsl, pa0, pa1);
            } else {
#pragma unroll
                for (int sl = 0; sl < SPS; ++sl) {
                    if (sl < nsl) {
                        const uint2 *fk = fr + (stored ? sl * KT * NB * LW : 0);
                        seg_mma<BITS, L, NB, LW, ACC, false>(c, A0[sl], A1[sl], fk, stored);
                        fresh = false;
                        if (--crem == 0) {  // this segment ends a scale group
                            flush();
                            crem = a.spg;
                            ++lg;
                        }
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(fempty + slot);
            if (++slot == nring) { slot = 0; ++round; }
        }
        if (nst > 0) {
            if (!fresh) flush();
            fold();
        }
        if (a.CS == 1) {
#pragma unroll
            for (int nb = 0; nb < NB; ++nb) {
                const int ml = nb * 4 + t;
                if (ml < mcnt) {
                    float *yr = a.y + (int64_t)(mc * 16 + ml) * a.N;
                    if (ok0) yr[row0] = acc0[nb];
                    if (ok1) yr[row1] = acc1[nb];
                }
            }
        } else {
#pragma unroll
            for (int nb = 0; nb < NB; ++nb) {
                const int ml = nb * 4 + t;
                if (ml < mcnt) {
                    red[pr * 16 + ml] = acc0[nb];
                    red[(pr + 8) * 16 + ml] = acc1[nb];
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

template <int BITS, int L, int NB, int LW, int GPS>
cudaError_t launch_typed(const GemvPlan &pl, const GemvArgs &a, const CUtensorMap &tm, bool xbf16,
                         cudaStream_t st) {
    if (xbf16)
        gemv_prep<BITS, L, NB, true><<<dim3(pl.n_eb, pl.nmc), 256, 0, st>>>(a);
    else
        gemv_prep<BITS, L, NB, false><<<dim3(pl.n_eb, pl.nmc), 256, 0, st>>>(a);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    auto kern = gemv_stream<BITS, L, NB, LW, GPS>;
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
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, kern, a, tm);
}

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

cudaError_t dispatch_gemv(const GemvPlan &pl, const GemvArgs &a, const CUtensorMap &tm, bool x_bf16,
                          cudaStream_t st, int64_t group) {
    // groups per 128-byte stage when the group size divides the stage, else 0
    const int stagek = kTileBytes * 8 / pl.bits;
    const int gps = (stagek % group == 0) ? (int)(stagek / group) : 0;
#define Q4_LW(B, LL, NBB, G)                                                                       \
    if constexpr (NBB == 1) {                                                                      \
        if (pl.lw == 8) return launch_typed<B, LL, NBB, 8, G>(pl, a, tm, x_bf16, st);             \
    }                                                                                              \
    return launch_typed<B, LL, NBB, 32, G>(pl, a, tm, x_bf16, st);
// per-group chains cost registers: kept for one column block, or two with at most 2 groups
#define Q4_GPS(B, LL, NBB, G1, G2)                                                                 \
    if (pl.bits == B && pl.L == LL && pl.NB == NBB) {                                              \
        if constexpr (NBB == 1 || (NBB == 2 && G1 <= 2)) {                                         \
            if (gps == G1) { Q4_LW(B, LL, NBB, G1) }                                               \
        }                                                                                          \
        if constexpr (G2 > 0 && NBB <= 2) {                                                        \
            if (gps == G2) { Q4_LW(B, LL, NBB, G2) }                                               \
        }                                                                                          \
        Q4_LW(B, LL, NBB, 0)                                                                       \
    }
#define Q4_GEMV(B, LL, NBB) Q4_GPS(B, LL, NBB, (LL == 16 ? 2 : LL == 8 ? 4 : 8), (LL == 16 ? 1 : 0))
    Q4_GEMV(4, 16, 1) Q4_GEMV(4, 16, 2) Q4_GEMV(4, 16, 4)
    Q4_GEMV(4, 8, 1) Q4_GEMV(4, 8, 2) Q4_GEMV(4, 8, 4)
    Q4_GEMV(4, 4, 1) Q4_GEMV(4, 4, 2) Q4_GEMV(4, 4, 4)
    Q4_GEMV(8, 16, 1) Q4_GEMV(8, 16, 2) Q4_GEMV(8, 16, 4)
    Q4_GEMV(8, 8, 1) Q4_GEMV(8, 8, 2) Q4_GEMV(8, 8, 4)
    Q4_GEMV(8, 4, 1) Q4_GEMV(8, 4, 2) Q4_GEMV(8, 4, 4)
#undef Q4_GEMV
#undef Q4_GPS
#undef Q4_LW
    return cudaErrorInvalidValue;
}



}  // namespace

bool gemv_plan(int64_t M, int64_t N, int64_t K, int bits, int64_t group, int sms, GemvPlan *pl) {
    GemvPlan p = {};
    p.bits = bits;
    if (K % 32 != 0 || group <= 0 || K % group != 0) return false;
    if (bits == 4)
        p.L = group % 128 == 0 ? 16 : group % 64 == 0 ? 8 : group % 32 == 0 ? 4 : 0;
    else
        p.L = group % 64 == 0 ? 16 : group % 32 == 0 ? 8 : group % 16 == 0 ? 4 : 0;
    if (!p.L) return false;
    if (K > ((int64_t)1 << 30) || N > ((int64_t)1 << 30) || M > ((int64_t)1 << 20)) return false;
    p.segk = 32 * p.L / bits;
    p.segs = (int)(K / p.segk);
    p.spg = (int)(group / p.segk);
    p.nmc = (int)((M + 15) / 16);
    const int mc0 = (int)(M < 16 ? M : 16);
    p.NB = mc0 > 8 ? 4 : mc0 > 4 ? 2 : 1;
    p.lw = (M == 1) ? 8 : 32;  // one row of x: only lanes 0..7 carry fragments
    p.T = (int)((N + 15) / 16);
    p.clusters = (int)((N + kRowsPerCta - 1) / kRowsPerCta);
    const int64_t rowbytes = K * bits / 8;
    p.stages_total = (int)((rowbytes + kTileBytes - 1) / kTileBytes);
    const int stagek = kTileBytes * 8 / bits;
    // k-block: <= 16 scale groups and <= 2048 k, in whole stages
    int64_t ebs = 16 * group / stagek;
    if (ebs > 2048 / stagek) ebs = 2048 / stagek;
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
    // ring stage = 16 KB of codes + the stage's fragments (slot_bytes, 16-aligned)
    const int kts = kTileBytes / (4 * p.L) * (p.segk / 16);
    p.slot_bytes = (int)align_up((size_t)kts * p.NB * p.lw * 8, 16);
    const size_t fixed = 1024 + 2 * (size_t)kRowsPerCta * kSG * 4 + (p.CS > 1 ? (size_t)kRowsPerCta * 16 * 4 : 0) +
                         16 + (4 * kMaxStages + 4) * 8;
    const size_t budget = 111 * 1024;  // two CTAs per SM
    int nr = (int)((budget - fixed) / (kPayloadBytes + p.slot_bytes));
    p.nst_ring = nr > kMaxStages ? kMaxStages : nr < 2 ? 2 : nr;
    p.smem_bytes = fixed + (size_t)p.nst_ring * (kPayloadBytes + p.slot_bytes);
    // workspace: fragments [mc][k-tile][nb][lw] x 8 bytes, then exponents [mc*16][n_eb]
    p.off_frag = 0;
    p.off_exp = align_up((size_t)p.nmc * (K / 16) * p.NB * p.lw * 8, 256);
    p.bytes = align_up(p.off_exp + (size_t)p.nmc * 16 * p.n_eb * 4, 256);
    *pl = p;
    return true;
}

cudaError_t launch_gemv(const GemvPlan &pl, const void *x, bool x_bf16, int64_t M,
                        const uint8_t *payload, const float *scales, int64_t N, int64_t K,
                        int64_t group, float *y, void *ws, uint32_t *status, cudaStream_t st) {
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
    a.frag = reinterpret_cast<const uint8_t *>(w + pl.off_frag);
    a.ebexp = reinterpret_cast<int *>(w + pl.off_exp);
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
    a.nst_ring = pl.nst_ring;
    a.slot_bytes = pl.slot_bytes;
    return dispatch_gemv(pl, a, tm, x_bf16, st, group);
}

}  // namespace q4
