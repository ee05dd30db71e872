// gemv.cu -- fused unpack -> dequant -> GEMV for decode (x in chunks of 16 rows).
//
// y[m][n] = sum_k x[m][k] * w'[n][k], w' = code * scale (pack()/unpack() of the
// "量化推理" page; the QuantizedMatmul of "Huit bits, puis quatre", which reads the
// codes in generation products, where one waits on memory). The packed weights are the
// whole cost, so the kernel is built around streaming them with as few instructions per
// byte as possible.
//
// Arithmetic: bf16 tensor-core products that are exact, accumulated in fp32 (warp-level
// mma.sync m16n8k16, bf16 x bf16 -> f32).
//   A = 16 weight rows x 16 k of codes as bf16, exact (|code| <= 127 < 2^8). An int4 byte
//       pair u (code + 8) becomes the bf16 128 + u by OR-ing the nibble into the mantissa
//       of 128.0, then one packed subtract of 136 gives the code; an int8 code c is
//       128 + (c & 127) minus (128 or 256, from its sign bit), again by bit masks and one
//       packed subtract. Two codes per 32-bit register.
//   B = 16 k x 8 columns of activation pieces: every fp32 activation is split exactly into
//       three bf16 values, x = hi + mid + lo (hi = x with its low 16 bits cleared, mid the
//       same of x - hi, lo = x - hi - mid, which has at most 8 significant bits), one B
//       column per piece (a bf16 activation is its own single piece).
//   C = fp32. Each product code * piece is exact in fp32; the tensor core sums them in
//       fp32. Because every product keeps its own exponent, the error of a sum is relative
//       to the sum of the magnitudes of its products, whatever the spread of |x|.
// Each scale group starts with a zero accumulator; when it ends (or the 128-byte stage
// ends, for groups longer than a stage) each lane multiplies its fp32 sums by the group's
// fp32 scale into fp32 totals. At the end the three piece columns of every activation
// row are added. The only roundings are those of fp32 sums.
//
// Structure (one wave: up to two CTAs per SM, a thread-block cluster of CS CTAs splits K):
//   a producer warp issues, per stage, one 2D TMA load of a 128-row x 128-byte tile of
//   the payload (128-byte swizzle) into a shared-memory ring guarded by full/empty
//   mbarriers, and loads each k-block's scales into double-buffered shared memory with
//   asynchronous copies (16 bytes wide when the rows of scales allow) one block ahead;
//   eight consumer warps decode and multiply.
//   One activation row (the decode case): the consumers build the pieces of their CTA's
//   K range into shared memory while the first payload tiles are in flight; there is no
//   second kernel and no workspace.
//   Several rows: gemv_prep writes the pieces once into the caller's workspace, in MMA
//   order, and the stream kernel (its programmatic dependent) copies each stage's tile
//   with a bulk copy into a second ring; the payload loads start before gemv_prep ends.
// Inside a group the order of k is permuted so that a lane builds its A fragment from its
// own shared-memory words; the pieces use the same permutation. Rows are permuted inside
// each 16-row tile so those reads are free of bank conflicts. The CS partial sums of a
// cluster meet in distributed shared memory in fixed rank order, so results do not depend
// on timing. Every wait is bounded; one that gives up sets Q4_STATUS_TIMEOUT.
#include <cuda.h>  // CUtensorMap and its enums (the encoder is fetched at run time)

#include "common.cuh"
#include "gemv_math.cuh"
#include "kernels.h"

namespace q4 {

namespace {

using namespace gm;

constexpr int kConsumers = 8;                      // consumer warps = 16-row tiles per CTA
constexpr int kConsumerThreads = 32 * kConsumers;
constexpr int kThreads = kConsumerThreads + 32;    // + 1 producer warp (the last warp)
constexpr int kRowsPerCta = 16 * kConsumers;       // 128
constexpr int kPayloadBytes = kTileBytes * kRowsPerCta;  // 16 KB of codes per stage
constexpr int kMaxStages = 6;
constexpr int kGroupsPerBlock = 8;                 // scale groups per k-block (target)
constexpr int kBlockK = 1024;                      // at most k per k-block
constexpr int kPrepSplit = 8;                      // gemv_prep CTAs per k-block (several rows of x)
constexpr int kSG = 12;                            // scale slots per row per k-block (<= 9 used,
                                                   // + up to 3 to keep 16-byte copies aligned)
constexpr int kInkMaxK = 4096;                     // k of one CTA's range whose pieces are built on
                                                   // chip (32 KB at 8 bytes per k)
constexpr int kSmemBudget2 = 115200;               // two CTAs per SM
constexpr int kSmemBudget1 = 232448 - 1024;        // one CTA per SM (227 KB opt-in maximum)
constexpr int kRedBytes = kRowsPerCta * 16 * 4;    // cluster partial sums, aliased on the ring

struct GemvArgs {
    const float *scales;
    const void *x;
    float *y;
    uint32_t *status;
    uint8_t *frag;        // workspace pieces: [mc][stage][fslot_bytes] (several rows of x)
    int M, N, K;
    int P;                // pieces per activation: 3 (fp32 x) or 1 (bf16 x)
    int segs;             // segments per weight row
    int spg;              // segments per scale group
    int scales_per_row;   // K / group
    int CS;               // CTAs per cluster = K splits
    int stages_total;     // 128-byte tiles per weight row (last may be partial)
    int stages_per_cta;
    int ebs;              // stages per k-block (scale block)
    int n_eb;
    int lw;               // piece lanes stored per (MMA, n8 block): 16 or 32
    int NB;               // n8 blocks of MMA columns per 16-row chunk of x
    int paired;           // pieces of two consecutive MMAs interleaved (16-byte reads)
    int nst_ring;         // ring depth
    int fslot_bytes;      // piece bytes of one stage
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

// Columns whose pieces are stored, and virtual rows of x that cover them.
Q4_DEVINL int stored_cols(int NB, int lw) { return (lw == 16 ? 4 : 8) * NB; }

// One CTA per (k-block eb, 16-row chunk mc of x): the pieces of the block in MMA order
// (several rows of x), zero columns for rows past M.
template <int BITS, int L, bool XBF16, bool HYB>
__global__ void __launch_bounds__(256) gemv_prep(const GemvArgs a) {
    grid_dep_launch();
    grid_dep_wait();  // x may be the output of the kernel before this one
    constexpr int STAGEK = kTileBytes * 8 / BITS;
    if constexpr (HYB) {
        // one row of x: each warp builds whole stage slots of the k-block (digits or pieces)
        const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
        const int s0 = blockIdx.x * a.ebs, s1 = min(s0 + a.ebs, a.stages_total);
        for (int s = s0 + warp; s < s1; s += 8)
            build_slot1<BITS, L, XBF16, false>(a.frag + (size_t)s * a.fslot_bytes, a.x, s * STAGEK, a.K, a.P, lane);
        return;
    }
    // several rows: kPrepSplit CTAs share a k-block (an item, 8 k of one row, per thread
    // or two), so the loads of x are in flight together
    const int eb = blockIdx.x / kPrepSplit, part = blockIdx.x % kPrepSplit, mc = blockIdx.y;
    const int mcnt = min(16, a.M - mc * 16);
    const int ncols = stored_cols(a.NB, a.lw);
    const int vrows = (ncols + a.P - 1) / a.P;
    const int k0 = eb * a.ebs * STAGEK;
    const int k1 = min(a.K, k0 + a.ebs * STAGEK);
    const int nu = (k1 - k0) / 8;  // 8-k units in the block (at most 128)
    const int u_lo = part * nu / kPrepSplit, nun = (part + 1) * nu / kPrepSplit - u_lo;
    uint2 *fbase = reinterpret_cast<uint2 *>(a.frag) + (size_t)mc * a.stages_total * (a.fslot_bytes / 8);
    for (int it = threadIdx.x; it < nun * vrows; it += blockDim.x) {
        const int vm = it / nun, u = u_lo + (it - vm * nun);
        const int k = k0 + 8 * u;
        float v[8];
        if (vm < mcnt) {
            load_x8<XBF16>(a.x, (int64_t)(mc * 16 + vm) * a.K + k, v);
        } else {
#pragma unroll
            for (int q = 0; q < 8; ++q) v[q] = 0.f;
        }
        const int s = k / STAGEK;
        frag_unit<BITS, L>(fbase + (size_t)s * (a.fslot_bytes / 8), k - s * STAGEK, vm, v, a.P, ncols, a.NB, a.lw,
                           a.paired != 0);
    }
}

// INK: the pieces of one row of x, or of two to four fp32 rows (one or two column blocks),
// are built by the consumers in shared memory (no workspace); otherwise they come from
// gemv_prep through a second ring. GPS: groups per stage
// when they divide it, 0 when the stage lies inside one group, -1 for any other group
// size (tracked segment by segment at run time).
// WIDE: one CTA per SM, so the registers of two (the plan's choice for up to four column
// blocks when the grid stays full; see gemv_plan)
template <int BITS, int L, int NB, int GPS, bool INK, bool XBF16, bool HYB, bool WIDE>
__global__ void __launch_bounds__(kThreads) __maxnreg__(NB >= 5 || WIDE ? 160 : 96)
gemv_stream(const GemvArgs a, const __grid_constant__ CUtensorMap tmap) {
    constexpr int SPS = kTileBytes / (4 * L);          // segments per stage
    constexpr int KTI = BITS == 4 ? L / 2 : L / 4;     // MMAs per segment
    constexpr int KTS = SPS * KTI;                     // MMAs per stage (16 int4, 8 int8)
    constexpr int WPT = L / 4;
    constexpr int STAGEK = kTileBytes * 8 / BITS;
    constexpr bool PAIRED = NB <= 2;
    static_assert(!INK || NB <= 2, "on-chip pieces cover at most two column blocks");
    static_assert(!HYB || (NB == 1 && GPS >= 0), "one row of x, regular groups");
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const int nring = a.nst_ring;
    uint8_t *slots = smem;                                   // codes: nring x 16 KB (1024-aligned)
    uint8_t *fslots = smem + nring * kPayloadBytes;          // pieces: ring slots, or the CTA's range
    const int nfrag = INK ? a.stages_per_cta : nring;
    float *scl = reinterpret_cast<float *>(fslots + nfrag * a.fslot_bytes);  // [2][128][kSG]
    uint64_t *full = reinterpret_cast<uint64_t *>(scl + 2 * kRowsPerCta * kSG);  // codes landed
    uint64_t *empty = full + kMaxStages;                                  // codes copied to registers
    uint64_t *ffull = empty + kMaxStages;                                 // pieces landed
    uint64_t *fempty = ffull + kMaxStages;                                // pieces no longer read
    uint64_t *sfull = fempty + kMaxStages;
    uint64_t *sempty = sfull + 2;
    float *red = reinterpret_cast<float *>(slots);                    // [128][16] per-CTA sums
    float *redc = reinterpret_cast<float *>(slots + kRedBytes);       // [128][8 * NB] piece columns

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
        // The first `primed` stages' pieces are copied once gemv_prep has finished, so that
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
        int sc_issued[2] = {0, 0};        // scale copies per buffer (phases of sfull)
        for (int ks = 0; ks < nst; ++ks) {
            const int s = st_lo + ks;
            if (eb_left == 0) {
                // stage the k-block's scales (all 32 lanes), one block ahead of the consumers
                if (ks > 0) ++eb;
                eb_left = min(a.ebs * (eb + 1), st_hi) - s;
                const int ebl = eb - eb_first, b = ebl & 1;
                if (ebl >= 2) {
                    // the consumers release this buffer only after the pieces of the
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
                ++sc_issued[b];
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
        // drain: every copy into this CTA's shared memory has landed before the CTA may
        // exit (only a wait that gave up can leave one in flight). Slot q received
        // ceil((nst - q) / nring) payload tiles and, without on-chip pieces, as many piece
        // tiles; the last phase of each barrier is the one to wait for.
        for (int q = 0; q < nring && q < nst; ++q) {
            const int n = (nst - q + nring - 1) / nring;
            (void)mbar_wait(full + q, (uint32_t)((n - 1) & 1));
            if constexpr (!INK) (void)mbar_wait(ffull + q, (uint32_t)((n - 1) & 1));
        }
        for (int b2 = 0; b2 < 2; ++b2)
            if (sc_issued[b2] > 0) (void)mbar_wait(sfull + b2, (uint32_t)((sc_issued[b2] - 1) & 1));
    } else {
        // ---------------- consumers ----------------
        const int g = lane >> 2, t = lane & 3;
        const int ct = threadIdx.x;  // 0..255
        // x may be the output of the kernel before this one, and y may still be read by it
        // (a no-op unless this grid was launched as a dependent)
        grid_dep_wait();
        if constexpr (INK && HYB) {
            // the B fragments of this CTA's stages (digits or pieces, per stage), one stage
            // per warp, built while the first payload tiles are in flight
            for (int ls = warp; ls < nst; ls += kConsumers)
                build_slot1<BITS, L, XBF16, false>(fslots + (size_t)ls * a.fslot_bytes, a.x, (st_lo + ls) * STAGEK,
                                                  a.K, a.P, lane);
            named_barrier_sync(1, kConsumerThreads);
        } else if constexpr (INK) {
            // pieces of this CTA's K range of the rows of x, built while the first payload
            // tiles are in flight (one item, 8 k of one row, per thread at a time, as in
            // gemv_prep); columns past the rows (and the lanes past the stored width, which
            // repeat these) are zero
            const int k_lo = st_lo * STAGEK, k_hi = min(st_hi * STAGEK, a.K);
            const int nu = max(k_hi - k_lo, 0) / 8;
            const int ncols = stored_cols(NB, a.lw);
            const int vrows = (ncols + a.P - 1) / a.P;
            uint2 *fbase = reinterpret_cast<uint2 *>(fslots);
            for (int it = ct; it < nu * vrows; it += kConsumerThreads) {
                const int vm = it / nu, u = it - vm * nu;
                float v[8];
                if (vm < a.M) {
                    load_x8<XBF16>(a.x, (int64_t)vm * a.K + k_lo + 8 * u, v);
                } else {
#pragma unroll
                    for (int q = 0; q < 8; ++q) v[q] = 0.f;
                }
                const int ls = (8 * u) / STAGEK;  // local stage
                frag_unit<BITS, L>(fbase + (size_t)ls * (a.fslot_bytes / 8), 8 * u - ls * STAGEK, vm, v, a.P, ncols,
                                   NB, a.lw, a.paired != 0);
            }
            named_barrier_sync(1, kConsumerThreads);
        }
        const int pr = 16 * warp + row_perm<L>(g);  // physical row of MMA row g in the CTA
        uint32_t aoff[SPS];
#pragma unroll
        for (int sl = 0; sl < SPS; ++sl) {
            const int off = sl * 4 * L + t * L;
            aoff[sl] = pr * kTileBytes + (((off >> 4) ^ (pr & 7)) << 4) + (off & 15);
        }
        const int lwr = a.lw;
        const int fl = lane & (lwr - 1);  // lanes past the stored width repeat lanes (their columns are unused)
        float ys0 = 0.f, ys1 = 0.f;  // one row of x: this lane's share of rows pr and pr + 8
        float cacc[NB][4], acc[NB][4];
#pragma unroll
        for (int nb = 0; nb < NB; ++nb)
#pragma unroll
            for (int e = 0; e < 4; ++e) cacc[nb][e] = acc[nb][e] = 0.f;
        int lg = (st_lo * SPS) / a.spg;                 // group of the next segment
        int crem = a.spg - (st_lo * SPS - lg * a.spg);  // segments left in that group
        int gA = 0, ng = 0, b = 0;
        const float *sb = scl;
        auto flush = [&](int q) {  // a group (or a stage) ends: scale its sums
            const float s0 = sb[pr * kSG + q], s1 = sb[(pr + 8) * kSG + q];
#pragma unroll
            for (int nb = 0; nb < NB; ++nb) {
                acc[nb][0] = fmaf(s0, cacc[nb][0], acc[nb][0]);
                acc[nb][1] = fmaf(s0, cacc[nb][1], acc[nb][1]);
                acc[nb][2] = fmaf(s1, cacc[nb][2], acc[nb][2]);
                acc[nb][3] = fmaf(s1, cacc[nb][3], acc[nb][3]);
                cacc[nb][0] = cacc[nb][1] = cacc[nb][2] = cacc[nb][3] = 0.f;
            }
        };
        int slot = 0, round = 0;
        int eb = eb_first, eb_left = 0;
        for (int ks = 0; ks < nst; ++ks) {
            const int s = st_lo + ks;
            if (eb_left == 0) {
                if (ks > 0) {
                    __syncwarp();
                    if (lane == 0) mbar_arrive(sempty + b);
                    ++eb;
                }
                eb_left = min(a.ebs * (eb + 1), st_hi) - s;
                const int ebl = eb - eb_first;
                b = ebl & 1;
                eb_groups(eb, gA, ng);
                sb = scl + b * kRowsPerCta * kSG + (vec16 ? (gA & 3) : 0);
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
            if constexpr (HYB) {
                const int qb = (GPS > 0 ? s * GPS : (s * SPS) / a.spg) - gA;  // first group, in the k-block
                const float *s0p = sb + pr * kSG + qb, *s1p = s0p + 8 * kSG;
                const int *hdr = reinterpret_cast<const int *>(fr + slot1_data<BITS>());
                if (hdr[0]) {
                    const float fl8 = digit_lane_factor<BITS>(hdr[1], t);
                    if (nsl == SPS)
                        stage1_digits<BITS, L, GPS, true>(A0, A1, fr, lane, s0p, s1p, nsl, fl8, ys0, ys1);
                    else
                        stage1_digits<BITS, L, GPS, false>(A0, A1, fr, lane, s0p, s1p, nsl, fl8, ys0, ys1);
                } else {
                    if (nsl == SPS)
                        stage1_pieces<BITS, L, GPS, true>(A0, A1, fr, lane, s0p, s1p, nsl, ys0, ys1);
                    else
                        stage1_pieces<BITS, L, GPS, false>(A0, A1, fr, lane, s0p, s1p, nsl, ys0, ys1);
                }
            } else if constexpr (GPS >= 0) {
                const int qb = (GPS > 0 ? s * GPS : (s * SPS) / a.spg) - gA;  // first group, in the k-block
                const float *s0p = sb + pr * kSG + qb, *s1p = s0p + 8 * kSG;
                const uint8_t *frl = fr + fl * (PAIRED ? 16 : 8);
                if (lwr == 16) {
                    if (nsl == SPS)
                        stage_fixed<BITS, L, NB, 16, GPS, true>(A0, A1, frl, s0p, s1p, nsl, acc);
                    else
                        stage_fixed<BITS, L, NB, 16, GPS, false>(A0, A1, frl, s0p, s1p, nsl, acc);
                } else {
                    if (nsl == SPS)
                        stage_fixed<BITS, L, NB, 32, GPS, true>(A0, A1, frl, s0p, s1p, nsl, acc);
                    else
                        stage_fixed<BITS, L, NB, 32, GPS, false>(A0, A1, frl, s0p, s1p, nsl, acc);
                }
            } else {
                uint4 bq[PAIRED ? NB : 1];
                const uint8_t *frl = fr + fl * (PAIRED ? 16 : 8);
#pragma unroll
                for (int i = 0; i < KTS; ++i) {
                    const int sl = i / KTI, j = i % KTI;
                    if (sl < nsl) {
                        uint32_t af[4];
                        unpack_a<BITS, L>(af, A0[sl], A1[sl], j);
#pragma unroll
                        for (int nb = 0; nb < NB; ++nb) {
                            uint32_t b0, b1;
                            if (lwr == 16)
                                load_b<NB, 16, PAIRED>(frl, i, nb, bq, b0, b1);
                            else
                                load_b<NB, 32, PAIRED>(frl, i, nb, bq, b0, b1);
                            mma_bf16(cacc[nb], af, b0, b1);
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
        if constexpr (HYB) {
            // one row of x: the four lanes of each row add their shares; lane 4g writes row
            // pr, lane 4g + 1 row pr + 8 (the partial sums of a K split go to the ring,
            // which every warp must be done with first)
            float r0 = ys0 + __shfl_xor_sync(0xffffffffu, ys0, 1);
            float r1 = ys1 + __shfl_xor_sync(0xffffffffu, ys1, 1);
            r0 += __shfl_xor_sync(0xffffffffu, r0, 2);
            r1 += __shfl_xor_sync(0xffffffffu, r1, 2);
            const int r = pr + 8 * (t & 1);
            const float v = (t & 1) ? r1 : r0;
            if (a.CS == 1) {
                const int n = cl * kRowsPerCta + r;
                if (t < 2 && n < a.N) a.y[n] = v;
            } else {
                named_barrier_sync(1, kConsumerThreads);
                if (t < 2) red[r * 16] = v;
            }
        } else {
        // add the pieces of each activation row: every warp writes its rows' piece columns
        // (column P * m + p) and sums its own rows; the ring is reused, so every warp must
        // be done with it first
        named_barrier_sync(1, kConsumerThreads);
        const int ncol = 8 * NB;
#pragma unroll
        for (int nb = 0; nb < NB; ++nb)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                redc[pr * ncol + 8 * nb + 2 * t + e] = acc[nb][e];
                redc[(pr + 8) * ncol + 8 * nb + 2 * t + e] = acc[nb][2 + e];
            }
        __syncwarp();
        for (int it = lane; it < 16 * mcnt; it += 32) {
            const int r = 16 * warp + (it & 15), m = it >> 4;
            const float *src = redc + r * ncol + a.P * m;
            float v = src[0];
            for (int p = 1; p < a.P; ++p) v += src[p];
            if (a.CS == 1) {
                const int n = cl * kRowsPerCta + r;
                if (n < a.N) a.y[(int64_t)(mc * 16 + m) * a.N + n] = v;
            } else {
                red[r * 16 + m] = v;
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

// early: the weights are static, so the call's first grid may start (and the stream
// kernel read payload and scales) while the previous kernel on the stream still runs.
// Every read of x, and every write, still waits for that kernel to finish.
template <int BITS, int L, int NB, int GPS, bool INK, bool XBF16, bool HYB = false, bool WIDE = false>
cudaError_t launch_typed(const GemvPlan &pl, const GemvArgs &a, const CUtensorMap &tm, bool x_bf16,
                         bool early, cudaStream_t st) {
    cudaError_t err;
    cudaLaunchAttribute pdl;
    pdl.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl.val.programmaticStreamSerializationAllowed = 1;
    // chunks of many rows of x (NB > 4) ignore the flag: their early start was measured
    // slower (a Llama-7B-shaped decode step at M = 16: 4.93 ms against 4.81 ms)
    if (NB > 4) early = false;
    if constexpr (!INK) {
        cudaLaunchConfig_t pc = {};
        pc.gridDim = dim3(HYB ? pl.n_eb : pl.n_eb * kPrepSplit, pl.nmc);
        pc.blockDim = dim3(256);
        pc.stream = st;
        pc.attrs = &pdl;
        pc.numAttrs = early ? 1 : 0;
        err = x_bf16 ? cudaLaunchKernelEx(&pc, gemv_prep<BITS, L, true, HYB>, a)
                     : cudaLaunchKernelEx(&pc, gemv_prep<BITS, L, false, HYB>, a);
        if (err != cudaSuccess) return err;
    }
    auto kern = gemv_stream<BITS, L, NB, GPS, INK, XBF16, HYB, WIDE>;
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
    if (pl.bits == B && pl.L == LL && pl.gps == G) {                                             \
        if (a.M > 1)                                                                             \
            return pl.NB == 2 ? launch_typed<B, LL, 2, G, true, false, false, true>(pl, a, tm, false, early, st) \
                              : launch_typed<B, LL, 1, G, true, false, false, true>(pl, a, tm, false, early, st); \
        return x_bf16 ? launch_typed<B, LL, 1, G, true, true, (G >= 0)>(pl, a, tm, true, early, st) \
                      : launch_typed<B, LL, 1, G, true, false, (G >= 0)>(pl, a, tm, false, early, st); \
    }
#define Q4_STAGED(B, LL, G)                                                                      \
    if (pl.bits == B && pl.L == LL && pl.gps == G) {                                             \
        if (pl.hyb) {                                                                            \
            if constexpr (G >= 0)                                                                \
                return x_bf16 ? launch_typed<B, LL, 1, (G >= 0 ? G : 0), false, true, true>(      \
                                    pl, a, tm, true, early, st)                                  \
                              : launch_typed<B, LL, 1, (G >= 0 ? G : 0), false, false, true>(     \
                                    pl, a, tm, false, early, st);                                \
        }                                                                                        \
        switch (pl.NB) {                                                                         \
            case 1:                                                                              \
                return pl.ctas_per_sm == 1                                                       \
                           ? launch_typed<B, LL, 1, G, false, false, false, true>(pl, a, tm, x_bf16, early, st) \
                           : launch_typed<B, LL, 1, G, false, false>(pl, a, tm, x_bf16, early, st);    \
            case 2:                                                                              \
                return pl.ctas_per_sm == 1                                                       \
                           ? launch_typed<B, LL, 2, G, false, false, false, true>(pl, a, tm, x_bf16, early, st) \
                           : launch_typed<B, LL, 2, G, false, false>(pl, a, tm, x_bf16, early, st);    \
            case 3:                                                                              \
                return pl.ctas_per_sm == 1                                                       \
                           ? launch_typed<B, LL, 3, G, false, false, false, true>(pl, a, tm, x_bf16, early, st) \
                           : launch_typed<B, LL, 3, G, false, false>(pl, a, tm, x_bf16, early, st);    \
            case 4:                                                                              \
                return pl.ctas_per_sm == 1                                                       \
                           ? launch_typed<B, LL, 4, G, false, false, false, true>(pl, a, tm, x_bf16, early, st) \
                           : launch_typed<B, LL, 4, G, false, false>(pl, a, tm, x_bf16, early, st);    \
            default: return launch_typed<B, LL, 6, G, false, false>(pl, a, tm, x_bf16, early, st); \
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

bool encode_payload_map(CUtensorMap *tm, const uint8_t *payload, int64_t N, int64_t K, int bits, int box_rows) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const uint64_t rowbytes = (uint64_t)K * bits / 8;
    const cuuint64_t dims[2] = {rowbytes, (cuuint64_t)N};
    const cuuint64_t strides[1] = {rowbytes};
    const cuuint32_t box[2] = {(cuuint32_t)kTileBytes, (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return enc(tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(payload), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool gemv_plan(int64_t M, int64_t N, int64_t K, int bits, int64_t group, bool x_bf16, int sms, GemvPlan *pl) {
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
    p.P = x_bf16 ? 1 : 3;
    p.segk = 32 * p.L / bits;
    p.segs = (int)(K / p.segk);
    p.spg = (int)(group / p.segk);
    p.nmc = (int)((M + 15) / 16);
    const int mc0 = (int)(M < 16 ? M : 16);
    const int ncols = p.P * mc0;  // MMA columns: one per piece of each row of x
    const int nbm = (ncols + 7) / 8;
    p.NB = nbm <= 4 ? nbm : 6;
    p.paired = p.NB <= 2;
    p.lw = (p.NB == 1 && ncols <= 4) ? 16 : 32;
    p.clusters = (int)((N + kRowsPerCta - 1) / kRowsPerCta);
    const int64_t rowbytes = K * bits / 8;
    p.stages_total = (int)((rowbytes + kTileBytes - 1) / kTileBytes);
    const int stagek = kTileBytes * 8 / bits;
    // k-block (scale staging unit): about kGroupsPerBlock scale groups and at most kBlockK
    // k, in whole stages
    int64_t ebs = kGroupsPerBlock * group / stagek;
    if (ebs > kBlockK / stagek) ebs = kBlockK / stagek;
    if (ebs < 1) ebs = 1;
    p.ebs = (int)ebs;
    p.n_eb = (p.stages_total + p.ebs - 1) / p.ebs;
    // many piece columns need a deep ring of large slots: one CTA per SM
    p.ctas_per_sm = p.NB >= 3 ? 1 : 2;
    // fp32 rows of x in one to four column blocks: one CTA per SM (the registers of two)
    // when the K split over a cluster can still be 2 or more, else two per SM at 96
    // registers, which keeps more CTAs in flight (measured, int4 g128 with static weights:
    // 4096x4096 M = 4 13.5 -> 8.6 us with one per SM; 11008x4096 M = 4 15.5 us with two
    // per SM, 18.7 with one; M = 8 23.7 -> 18.1 us with two)
    const int64_t blocks0 = (int64_t)p.clusters * p.nmc;
    if (p.NB <= 4 && M > 1 && !x_bf16 && blocks0 > 0) p.ctas_per_sm = sms / blocks0 >= 2 ? 1 : 2;
    const size_t budget = p.ctas_per_sm == 2 ? kSmemBudget2 : kSmemBudget1;
    // split K over a cluster so that the grid is one wave
    const int64_t slots = (int64_t)sms * p.ctas_per_sm;
    const int64_t blocks = (int64_t)p.clusters * p.nmc;
    int64_t cs = slots / (blocks > 0 ? blocks : 1);
    if (cs > 8) cs = 8;
    if (cs > p.stages_total / 2) cs = p.stages_total / 2;
    p.CS = cs < 1 ? 1 : (int)cs;
    p.stages_per_cta = (p.stages_total + p.CS - 1) / p.CS;
    const int kts = bits == 4 ? 16 : 8;  // MMAs per stage
    // one row of x: 16 piece lanes, built on chip when the CTA's K range fits; with
    // regular groups each stage's slot holds digits or pieces plus a header
    p.ink = M == 1 && (int64_t)p.stages_per_cta * stagek <= kInkMaxK;
    if (p.ink) p.lw = 16;
    p.hyb = M == 1 && p.gps >= 0;
    p.fslot_bytes = p.hyb ? (bits == 4 ? slot1_bytes<4>() : slot1_bytes<8>()) : kts * p.NB * p.lw * 8;
    const size_t fixed = 1024 + 2 * (size_t)kRowsPerCta * kSG * 4 + (4 * kMaxStages + 4) * 8;
    // two to four fp32 rows at one CTA per SM: their pieces are built on chip too when the
    // CTA's K range and its slots fit (no gemv_prep launch, no workspace round trip)
    if (!p.ink && M > 1 && M <= 4 && !x_bf16 && p.NB <= 2 && p.ctas_per_sm == 1 &&
        (int64_t)p.stages_per_cta * stagek <= kInkMaxK &&
        budget >= fixed + (size_t)p.stages_per_cta * p.fslot_bytes + 2 * (size_t)kPayloadBytes)
        p.ink = true;
    int nr;
    if (p.ink) {
        const size_t frag = (size_t)p.stages_per_cta * p.fslot_bytes;
        nr = (int)((budget - fixed - frag) / kPayloadBytes);
        p.nst_ring = nr > kMaxStages ? kMaxStages : nr < 2 ? 2 : nr;
        p.smem_bytes = fixed + frag + (size_t)p.nst_ring * kPayloadBytes;
    } else {
        nr = (int)((budget - fixed) / (kPayloadBytes + p.fslot_bytes));
        p.nst_ring = nr > kMaxStages ? kMaxStages : nr < 2 ? 2 : nr;
        p.smem_bytes = fixed + (size_t)p.nst_ring * (kPayloadBytes + p.fslot_bytes);
    }
    // the end of the kernel reuses the code ring: [128][16] sums + [128][8 * NB] columns
    if ((size_t)kRedBytes + (size_t)kRowsPerCta * 8 * p.NB * 4 > (size_t)p.nst_ring * kPayloadBytes) return false;
    // workspace (several rows of x): pieces [mc][stage][fslot_bytes]
    if (p.ink) {
        p.off_frag = p.bytes = 0;
    } else {
        p.off_frag = 0;
        p.bytes = align_up((size_t)p.nmc * p.stages_total * p.fslot_bytes, 256);
    }
    *pl = p;
    return true;
}

cudaError_t launch_gemv(const GemvPlan &pl, const void *x, bool x_bf16, int64_t M,
                        const uint8_t *payload, const float *scales, int64_t N, int64_t K,
                        int64_t group, float *y, void *ws, uint32_t *status, bool weights_static,
                        cudaStream_t st) {
    if (!encode_fn()) return cudaErrorNotSupported;
    CUtensorMap tm;
    if (!encode_payload_map(&tm, payload, N, K, pl.bits, kRowsPerCta)) return cudaErrorInvalidValue;
    char *w = static_cast<char *>(ws);
    GemvArgs a;
    a.scales = scales;
    a.x = x;
    a.y = y;
    a.status = status;
    a.frag = w ? reinterpret_cast<uint8_t *>(w + pl.off_frag) : nullptr;
    a.M = (int)M;
    a.N = (int)N;
    a.K = (int)K;
    a.P = pl.P;
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
