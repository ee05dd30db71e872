// gemv.cu -- fused unpack -> dequant -> GEMV for decode (x in chunks of 16 rows).
//
// y[m][n] = sum_k x[m][k] * w'[n][k], w' = code * scale (pack()/unpack() of the
// "量化推理" page; the QuantizedMatmul of "Huit bits, puis quatre", which reads the
// codes in generation products, where one waits on memory). The weight stream is the
// whole cost, so it is moved by the Tensor Memory Accelerator: a producer warp issues
// 2D TMA loads of 128-row x 128-byte tiles of the packed codes (128-byte swizzle) into a
// 4-stage shared-memory ring guarded by full/empty mbarriers, and 8 consumer warps
// decode and multiply. In-flight bytes no longer cost registers: 64 KB per CTA.
//
// Tensor cores (warp-level mma.sync m16n8k16, fp16 operands, fp32 accumulation):
//   A = 16 weight rows x 16 k of CODES, exact in fp16 (|code| <= 127).
//   B = 16 k x 8 columns of activations. Every activation row m is split exactly into
//       x' = hi + lo, hi = fp16(x'), lo = fp16(x' - hi) (22 significant bits), after a
//       power-of-two rescale x' = x * 2^-e that puts the largest |x| of the staged range
//       in [2^14, 2^15): no overflow, and the dropped part is below 2^-22 |x|.
//   Columns 2c and 2c+1 of B hold hi and lo of one activation row, so one lane owns
//   both partial sums of the same (weight row, m) in c0/c1 (and c2/c3).
//   When a scale group ends, the lane multiplies the partial sum by the group's fp32
//   scale and adds it to an fp32 accumulator; no arithmetic on w' is done in fp16.
// Inside a group the order of k is permuted so that a lane builds its A fragment from
// one shared-memory read; the staged B fragments use the same permutation. Rows are
// permuted inside each 16-row tile so that those reads are free of bank conflicts
// under the 128-byte swizzle.
//
// Work decomposition:
//   CTA = 8 consumer warps (warp w owns rows 16w..16w+15 of the CTA's 128) + 1
//   producer warp. A thread-block cluster of CS CTAs splits K into CS contiguous
//   ranges (CTA rank c takes range c). Each CTA stages the B fragments of its range of
//   x in shared memory (in phases when the range is long).
//   With CS > 1 the partial sums meet in distributed shared memory: after a cluster
//   barrier, CTA c adds the CS partials of its 128/CS rows in rank order and writes y.
// Everything happens in one kernel launch: no workspace, no atomics, no global fences,
// and the result does not depend on timing (fixed summation order). Every mbarrier wait
// is bounded; a wait that gives up sets Q4_STATUS_TIMEOUT in the optional status word.
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
constexpr int kStageBytes = kTileBytes * kRowsPerCta;  // 16 KB per stage
constexpr int kStages = 4;
constexpr int kFragBudget = 32 * 1024;             // shared memory for staged x per phase

struct GemvArgs {
    const float *scales;
    const void *x;
    float *y;
    uint32_t *status;
    int M, N, K;
    int segs;            // segments per weight row = K / segk
    int spg;             // segments per scale group
    int scales_per_row;  // K / group
    int CS;              // CTAs per cluster = K splits
    int stages_total;    // 128-byte tiles per weight row (last may be partial)
    int stages_per_cta;  // tiles per CTA's K range
    int phase_stages;    // tiles of x staged at a time
};

Q4_DEVINL void consumers_sync() { named_barrier_sync(1, kConsumerThreads); }

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

// x * 2^-e exactly for any e the staging can produce (|e| up to ~165).
Q4_DEVINL float pow2(int e) {  // 2^e, e in [-126, 127]
    return __int_as_float((e + 127) << 23);
}

// ---- staging of the B fragments of x for segments [s0, s1) ---------------------------
// Fragment layout in shared memory: [segment][nb][j][lane] of uint2 = (b0b1, b2b3).
// Every x value of the range is loaded once, in one round trip: a thread keeps up to
// IPT work items (8 values) in registers while the per-row maximum is reduced
// (shared-memory atomicMax on the magnitude bits); items beyond IPT per thread are re-read.

template <int BITS, bool XBF16, int BLK>
Q4_DEVINL void load_item(const GemvArgs &a, int mc, int k0, int nblk, int it, float (&v)[BLK], int &ml) {
    ml = it / nblk;
    const int blk = it - ml * nblk;
    const int64_t xb = (int64_t)(mc * 16 + ml) * a.K + k0 + blk * BLK;
    float t4[4];
    load_x4<XBF16>(a.x, xb, t4);
#pragma unroll
    for (int q = 0; q < 4; ++q) v[q] = t4[q];
    if constexpr (BLK == 8) {
        load_x4<XBF16>(a.x, xb + 4, t4);
#pragma unroll
        for (int q = 0; q < 4; ++q) v[4 + q] = t4[q];
    }
}

template <int BITS, int L, int NB, bool XBF16>
Q4_DEVINL void stage_x(const GemvArgs &a, int mc, int s0, int s1, uint2 *frag, int *e_sh,
                       uint32_t *mx_sh) {
    constexpr int SEGK = 32 * L / BITS;
    constexpr int KT = SEGK / 16;
    constexpr int BLK = BITS == 4 ? 8 : 4;  // k per work item
    constexpr int kIPT = 8 / BLK;
    const int mcnt = min(16, a.M - mc * 16);
    const int k0 = s0 * SEGK, nk = (s1 - s0) * SEGK;
    const int nblk = nk / BLK;
    const int items = nblk * mcnt;
    if (threadIdx.x < 16) mx_sh[threadIdx.x] = 0u;
    consumers_sync();
    // (a) load (kept in registers) + per-row max of |x|
    float v[kIPT][BLK];
    int mlr[kIPT];
#pragma unroll
    for (int q = 0; q < kIPT; ++q) {
        const int it = threadIdx.x + q * kConsumerThreads;
        mlr[q] = -1;
        if (it < items) load_item<BITS, XBF16, BLK>(a, mc, k0, nblk, it, v[q], mlr[q]);
    }
#pragma unroll
    for (int q = 0; q < kIPT; ++q) {
        if (mlr[q] >= 0) {
            uint32_t m = 0;
#pragma unroll
            for (int i = 0; i < BLK; ++i) m = max(m, __float_as_uint(v[q][i]) & 0x7fffffffu);
            atomicMax(mx_sh + mlr[q], m);
        }
    }
    for (int it = threadIdx.x + kIPT * kConsumerThreads; it < items; it += kConsumerThreads) {
        float w[BLK];
        int ml;
        load_item<BITS, XBF16, BLK>(a, mc, k0, nblk, it, w, ml);
        uint32_t m = 0;
#pragma unroll
        for (int i = 0; i < BLK; ++i) m = max(m, __float_as_uint(w[i]) & 0x7fffffffu);
        atomicMax(mx_sh + ml, m);
    }
    consumers_sync();
    if (threadIdx.x < 16) {
        const uint32_t mx = mx_sh[threadIdx.x];
        int e = 0;
        if (mx != 0 && mx < 0x7f800000u) {
            int E;
            frexpf(__uint_as_float(mx), &E);  // max|x| in [2^(E-1), 2^E)
            e = E - 15;                        // -> max|x| * 2^-e in [2^14, 2^15)
        }
        e_sh[threadIdx.x] = e;
    }
    consumers_sync();
    // (b) rescale, split, scatter into fragment order
    auto emit = [&](const float (&xv)[BLK], int ml, int it) {
        const int blk = it - ml * nblk;
        const int e = e_sh[ml];
        // x * 2^-e as two exact power-of-two multiplications (2^-e may leave fp32 range)
        const int e1 = min(max(-e, -126), 127);
        const float f1 = pow2(e1), f2 = pow2(min(max(-e - e1, -126), 127));
        float vv[BLK];
#pragma unroll
        for (int q = 0; q < BLK; ++q) vv[q] = (xv[q] * f1) * f2;
        const int kl = blk * BLK;  // k offset inside the staged range
        const int sl = kl / SEGK, within = kl - sl * SEGK;
        const int nb = (ml >> 2), lane_hi = 8 * (ml & 3);
        if constexpr (BITS == 4) {
            // the 8 values are word w of lane quad t: j = 2w takes k {0,4 | 1,5},
            // j = 2w+1 takes k {2,6 | 3,7}
            const int t = within / (2 * L), w = (within % (2 * L)) / 8;
            uint32_t h01, l01, h45, l45, h23, l23, h67, l67;
            split2(vv[0], vv[1], h01, l01);
            split2(vv[4], vv[5], h45, l45);
            split2(vv[2], vv[3], h23, l23);
            split2(vv[6], vv[7], h67, l67);
            uint2 *f0 = frag + ((sl * NB + nb) * KT + 2 * w) * 32 + lane_hi + t;
            uint2 *f1p = f0 + 32;  // j = 2w + 1
            f0[0] = make_uint2(pack_lo_halves(h01, h45), pack_hi_halves(h01, h45));
            f0[4] = make_uint2(pack_lo_halves(l01, l45), pack_hi_halves(l01, l45));
            f1p[0] = make_uint2(pack_lo_halves(h23, h67), pack_hi_halves(h23, h67));
            f1p[4] = make_uint2(pack_lo_halves(l23, l67), pack_hi_halves(l23, l67));
        } else {
            // the 4 values are word j of lane quad t, in natural order
            const int t = within / L, j = (within % L) / 4;
            uint32_t h01, l01, h23, l23;
            split2(vv[0], vv[1], h01, l01);
            split2(vv[2], vv[3], h23, l23);
            uint2 *f0 = frag + ((sl * NB + nb) * KT + j) * 32 + lane_hi + t;
            f0[0] = make_uint2(h01, h23);
            f0[4] = make_uint2(l01, l23);
        }
    };
#pragma unroll
    for (int q = 0; q < kIPT; ++q)
        if (mlr[q] >= 0) emit(v[q], mlr[q], threadIdx.x + q * kConsumerThreads);
    for (int it = threadIdx.x + kIPT * kConsumerThreads; it < items; it += kConsumerThreads) {
        float w[BLK];
        int ml;
        load_item<BITS, XBF16, BLK>(a, mc, k0, nblk, it, w, ml);
        emit(w, ml, it);
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

// L bytes of row r (0..127) of a swizzled stage, at byte offset `off` of the row.
template <int L>
Q4_DEVINL void lds_row(uint32_t (&dst)[L / 4], const uint8_t *stage, int r, int off) {
    const int chunk = off >> 4, within = off & 15;
    const uint8_t *p = stage + r * kTileBytes + ((chunk ^ (r & 7)) << 4) + within;
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

template <int BITS, int L, int NB, bool XBF16>
__global__ void __launch_bounds__(kThreads, 2)
gemv_tma_kernel(const GemvArgs a, const __grid_constant__ CUtensorMap tmap) {
    constexpr int SEGK = 32 * L / BITS;
    constexpr int KT = SEGK / 16;
    constexpr int WPT = L / 4;
    constexpr int SPS = kTileBytes / (4 * L);  // segments per stage
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint8_t *stages = smem;
    uint2 *frag = reinterpret_cast<uint2 *>(smem + kStages * kStageBytes);
    const size_t frag_bytes = (size_t)a.phase_stages * SPS * NB * KT * 32 * sizeof(uint2);
    float *red = reinterpret_cast<float *>(smem + kStages * kStageBytes + frag_bytes);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + kStages * kStageBytes + frag_bytes +
                                                  (a.CS > 1 ? kRowsPerCta * 16 * sizeof(float) : 0));
    uint64_t *empty = full + kStages;
    __shared__ int e_sh[16];
    __shared__ uint32_t mx_sh[16];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int crank = (int)(blockIdx.x % (unsigned)a.CS);
    const int cl = (int)(blockIdx.x / (unsigned)a.CS);
    const int mc = blockIdx.y;
    const int mcnt = min(16, a.M - mc * 16);
    const int st_lo = crank * a.stages_per_cta;
    const int st_hi = min(st_lo + a.stages_per_cta, a.stages_total);
    const int nst = max(st_hi - st_lo, 0);
    const int seg_hi = min(st_hi * SPS, a.segs);

    if (threadIdx.x == 0) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(full + i, 1);
            mbar_init(empty + i, kConsumers);
        }
        fence_barrier_init();
    }
    __syncthreads();

    bool timed_out = false;
    if (warp == kConsumers) {
        // ---------------- producer: one lane streams the CTA's tiles ----------------
        if (lane == 0) {
            for (int ks = 0; ks < nst; ++ks) {
                const int slot = ks % kStages;
                if (ks >= kStages && !timed_out)
                    timed_out = !mbar_wait(empty + slot, (uint32_t)((ks / kStages - 1) & 1));
                if (timed_out) break;
                mbar_arrive_expect_tx(full + slot, kStageBytes);
                tma_load_2d(stages + slot * kStageBytes, &tmap, full + slot, (st_lo + ks) * kTileBytes,
                            cl * kRowsPerCta);
            }
        }
    } else {
        // ---------------- consumers ----------------
        const int g = lane >> 2, t = lane & 3;
        const int pr = 16 * warp + row_perm<L>(g);  // physical row of MMA row g in the CTA
        const int row0 = cl * kRowsPerCta + pr, row1 = row0 + 8;
        const bool ok0 = row0 < a.N, ok1 = row1 < a.N;
        const float *s0p = a.scales + (size_t)(ok0 ? row0 : 0) * a.scales_per_row;
        const float *s1p = a.scales + (size_t)(ok1 ? row1 : 0) * a.scales_per_row;
        bool colok[NB];
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) colok[nb] = nb * 4 + (g >> 1) < mcnt;
        float acc0[NB], acc1[NB];
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) acc0[nb] = acc1[nb] = 0.f;

        // scale bookkeeping without division: group of the next segment to prefetch
        const int seg_lo = st_lo * SPS;
        int lg = seg_lo / a.spg, lrem = a.spg - (seg_lo - lg * a.spg);
        int crem = lrem;
        float sc0[SPS], sc1[SPS];
        auto fetch_scales = [&](int stg) {  // scales of the SPS segments of stage stg
#pragma unroll
            for (int sl = 0; sl < SPS; ++sl) {
                const int sg = stg * SPS + sl;
                if (sg < seg_hi) {
                    sc0[sl] = ok0 ? __ldg(s0p + lg) : 0.f;
                    sc1[sl] = ok1 ? __ldg(s1p + lg) : 0.f;
                    if (--lrem == 0) { ++lg; lrem = a.spg; }
                }
            }
        };

        for (int ph = 0; ph < nst; ph += a.phase_stages) {
            const int ph_end = min(ph + a.phase_stages, nst);
            consumers_sync();  // the previous phase's fragments are no longer read
            stage_x<BITS, L, NB, XBF16>(a, mc, (st_lo + ph) * SPS, min((st_lo + ph_end) * SPS, a.segs), frag,
                                        e_sh, mx_sh);
            consumers_sync();  // every warp's fragments are written before any warp reads them
            float pa0[NB], pa1[NB], c[NB][4];
#pragma unroll
            for (int nb = 0; nb < NB; ++nb) {
                pa0[nb] = pa1[nb] = 0.f;
                c[nb][0] = c[nb][1] = c[nb][2] = c[nb][3] = 0.f;
            }
            for (int ks = ph; ks < ph_end; ++ks) {
                const int slot = ks % kStages;
                fetch_scales(st_lo + ks);  // in flight while waiting for the tile
                if (!timed_out) timed_out = !mbar_wait(full + slot, (uint32_t)((ks / kStages) & 1));
                const uint8_t *stg = stages + slot * kStageBytes;
#pragma unroll
                for (int sl = 0; sl < SPS; ++sl) {
                    const int sgl = (ks - ph) * SPS + sl;  // segment index inside the phase
                    if ((st_lo + ks) * SPS + sl < seg_hi) {
                        uint32_t A0[WPT], A1[WPT];
                        lds_row<L>(A0, stg, pr, sl * 4 * L + t * L);
                        lds_row<L>(A1, stg, pr + 8, sl * 4 * L + t * L);
                        const uint2 *fb = frag + (int64_t)sgl * NB * KT * 32 + lane;
#pragma unroll
                        for (int j = 0; j < KT; ++j) {
                            uint32_t af[4];
                            unpack_a<BITS, L>(af, A0, A1, j);
#pragma unroll
                            for (int nb = 0; nb < NB; ++nb) {
                                uint2 b = make_uint2(0u, 0u);
                                if (colok[nb]) b = fb[(nb * KT + j) * 32];
                                mma_f16_16816(c[nb], af, b.x, b.y);
                            }
                        }
                        const bool group_end = --crem == 0;
                        if (group_end) crem = a.spg;
                        const bool last = (st_lo + ks) * SPS + sl + 1 == seg_hi || (ks + 1 == ph_end && sl + 1 == SPS);
                        if (group_end || last) {
#pragma unroll
                            for (int nb = 0; nb < NB; ++nb) {
                                pa0[nb] = fmaf(sc0[sl], c[nb][0] + c[nb][1], pa0[nb]);
                                pa1[nb] = fmaf(sc1[sl], c[nb][2] + c[nb][3], pa1[nb]);
                                c[nb][0] = c[nb][1] = c[nb][2] = c[nb][3] = 0.f;
                            }
                        }
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(empty + slot);
            }
            // undo this phase's activation rescale: acc += 2^e * partial (exact scaling)
#pragma unroll
            for (int nb = 0; nb < NB; ++nb) {
                const int ml = nb * 4 + t;
                const int e = ml < mcnt ? e_sh[ml] : 0;
                acc0[nb] += ldexpf(pa0[nb], e);
                acc1[nb] += ldexpf(pa1[nb], e);
            }
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
    const int rows_per = kRowsPerCta / a.CS;
    const int items = rows_per * mcnt;
    for (int it = threadIdx.x; it < items; it += kThreads) {
        const int rl = crank * rows_per + it / mcnt;  // row within the cluster's 128
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

template <int BITS, int L, int NB, bool XBF16>
cudaError_t launch_typed(const GemvPlan &pl, const GemvArgs &a, const CUtensorMap &tm, cudaStream_t st) {
    auto kern = gemv_tma_kernel<BITS, L, NB, XBF16>;
    const size_t smem = pl.smem_bytes;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    err = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (err != cudaSuccess) return err;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(pl.clusters * pl.CS, pl.nmc);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = pl.CS;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, a, tm);
}

template <int BITS, int L, int NB>
cudaError_t launch_x(const GemvPlan &pl, const GemvArgs &a, const CUtensorMap &tm, bool xbf16, cudaStream_t st) {
    return xbf16 ? launch_typed<BITS, L, NB, true>(pl, a, tm, st) : launch_typed<BITS, L, NB, false>(pl, a, tm, st);
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
    p.D = 0;
    p.T = (int)((N + 15) / 16);
    p.clusters = (int)((N + kRowsPerCta - 1) / kRowsPerCta);
    const int64_t rowbytes = K * bits / 8;
    p.stages_total = (int)((rowbytes + kTileBytes - 1) / kTileBytes);
    // split K over a cluster until about two CTAs per SM are busy
    const int64_t want = (int64_t)sms * 2;
    p.CS = 1;
    while (p.CS < 8 && (int64_t)p.clusters * p.CS * p.nmc < want && p.stages_total >= 2 * p.CS * 2) p.CS *= 2;
    p.stages_per_cta = (p.stages_total + p.CS - 1) / p.CS;
    const int sps = kTileBytes / (4 * p.L);
    const int kt = p.segk / 16;
    const size_t per_stage = (size_t)sps * p.NB * kt * 32 * 8;
    int ps = (int)(kFragBudget / per_stage);
    if (ps < 1) ps = 1;
    p.phase_stages = ps < p.stages_per_cta ? ps : p.stages_per_cta;
    p.seg_per_cta = p.stages_per_cta * sps;
    p.phase_segs = p.phase_stages * sps;
    p.smem_bytes = 1024 + (size_t)kStages * kStageBytes + (size_t)p.phase_stages * per_stage +
                   (p.CS > 1 ? (size_t)kRowsPerCta * 16 * sizeof(float) : 0) + 2 * kStages * sizeof(uint64_t);
    p.bytes = 0;  // no global workspace
    *pl = p;
    return true;
}

cudaError_t launch_gemv(const GemvPlan &pl, const void *x, bool x_bf16, int64_t M,
                        const uint8_t *payload, const float *scales, int64_t N, int64_t K,
                        int64_t group, float *y, uint32_t *status, cudaStream_t st) {
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
    GemvArgs a;
    a.scales = scales;
    a.x = x;
    a.y = y;
    a.status = status;
    a.M = (int)M;
    a.N = (int)N;
    a.K = (int)K;
    a.segs = pl.segs;
    a.spg = pl.spg;
    a.scales_per_row = (int)(K / group);
    a.CS = pl.CS;
    a.stages_total = pl.stages_total;
    a.stages_per_cta = pl.stages_per_cta;
    a.phase_stages = pl.phase_stages;
#define Q4_GEMV(B, LL, NBB) \
    if (pl.bits == B && pl.L == LL && pl.NB == NBB) return launch_x<B, LL, NBB>(pl, a, tm, x_bf16, st);
    Q4_GEMV(4, 16, 1) Q4_GEMV(4, 16, 2) Q4_GEMV(4, 16, 4)
    Q4_GEMV(4, 8, 1) Q4_GEMV(4, 8, 2) Q4_GEMV(4, 8, 4)
    Q4_GEMV(4, 4, 1) Q4_GEMV(4, 4, 2) Q4_GEMV(4, 4, 4)
    Q4_GEMV(8, 16, 1) Q4_GEMV(8, 16, 2) Q4_GEMV(8, 16, 4)
    Q4_GEMV(8, 8, 1) Q4_GEMV(8, 8, 2) Q4_GEMV(8, 8, 4)
    Q4_GEMV(8, 4, 1) Q4_GEMV(8, 4, 2) Q4_GEMV(8, 4, 4)
#undef Q4_GEMV
    return cudaErrorInvalidValue;
}

}  // namespace q4
