// prefill.cu -- the quantized matmul for many rows of bf16 activations (prefill), on the
// 5th-generation tensor cores.
//
// y[m][n] = sum_k x[m][k] * w'[n][k], w' = code * scale (the QuantizedMatmul of "Huit bits,
// puis quatre", section "Ranger des entiers dans des f32", in the case the page calls
// "where one computes more than one reads"). Codes and activations meet in tcgen05.mma
// (kind::f16, bf16 operands, fp32 accumulation in tensor memory):
//   A = 128 weight rows x 64 k of CODES as bf16 (exact: |code| <= 127), dequantized from
//       the payload into shared memory in the canonical K-major 128-byte-swizzle layout;
//   B = 256 activation rows x 64 k of x (bf16 as given), loaded by TMA with the same swizzle;
//   D = 128 lanes (weight rows) x 256 columns (activation rows) of fp32 in tensor memory.
// The scale is never folded into the bf16 operand (bf16(code * scale) would lose 16 bits):
// each scale group accumulates into its own tensor-memory buffer (two, alternating), and
// epilogue warps add scale * partial into fp32 registers ("promotion"), so the result is
// the fp32 product of exact codes and activations, rounded only by fp32 sums.
//
// Warp roles (512 threads, one CTA per SM, persistent over output tiles):
//   warp 0      TMA producer: x tile (256 x 64 bf16) and payload tile (128 rows) per k-step
//               into a 4-deep ring (full/empty mbarriers);
//   warp 1      allocates tensor memory; one lane issues the MMAs (4 per k-step) and the
//               tcgen05.commit arrivals that free ring slots and publish finished groups;
//   warps 2-5   dequantize the payload tile (one row per thread) into a 3-deep ring of A
//               tiles, made visible to the tensor core with fence.proxy.async (warps 6-7
//               have no role: they fill the second warpgroup);
//   warps 8-15  epilogue: warp w reads tensor-memory lanes 32*(w%4).. and 128 of the 256
//               columns, keeps them as fp32 accumulators, stores y at the end of a tile.
// Registers move from the first two warpgroups to the epilogue ones (setmaxnreg).
// With one scale per output channel (one group per tile) the scale is applied once at the
// end, the epilogue needs no accumulators and 4 warps (10-13), and warps 2-9 dequantize
// (consecutive threads take consecutive 16-byte chunks of the payload tile).
// Every wait is bounded (about one second); one that gives up sets Q4_STATUS_TIMEOUT in the
// status word, and the roles run to completion without further waits.
#include <cuda.h>

#include "common.cuh"
#include "kernels.h"

namespace q4 {

namespace {

constexpr int kBM = 128;          // weight rows per tile (MMA M)
constexpr int kBN = 256;          // activation rows per tile (MMA N)
constexpr int kBK = 64;           // k per step: one 128-byte swizzle row of bf16
constexpr int kStages = 4;        // x + payload ring
constexpr int kAStages = 3;       // dequantized A ring
constexpr int kThreads = 512;     // grouped scales: TMA, MMA, 4 dequantizing, 2 idle, 8 epilogue warps
// Grouped scales: the kernel launches at kRegsLaunch registers a thread; the first two
// warpgroups (TMA, MMA, dequantizing) give theirs down to kRegsLow and the two epilogue
// warpgroups (128 fp32 accumulators a thread) take kRegsHigh: 256 * 64 + 256 * 192 is
// exactly the 512 * 128 the block holds, so every increase is served.
constexpr int kRegsLaunch = 128, kRegsLow = 64, kRegsHigh = 192;
static_assert(4 * 32 * 2 * kRegsLow + 4 * 32 * 2 * kRegsHigh == kThreads * kRegsLaunch, "register split");
constexpr int kThreadsPC = 448;   // one scale per output channel: TMA, MMA, 8 dequantizing, 4 epilogue
constexpr int kXBytes = kBN * kBK * 2;        // 32 KB
constexpr int kABytes = kBM * kBK * 2;        // 16 KB
constexpr int kPBytesMax = kBM * kBK;         // 8 KB (int8); int4 uses half
constexpr int kTmemCols = 512;                // two D buffers of 256 columns


struct PrefillArgs {
    const float *scales;
    float *y;
    uint32_t *status;
    int M, N, K;
    int scales_per_row;   // K / group
    int kpg;              // k-steps per scale group
    int ksteps;           // K / kBK
    int tiles_n, tiles;   // output tiles: (N / 128) x (M / 256), n fastest
    int full_items;       // items that are whole tiles (a multiple of the grid)
    int split;            // the remaining tiles are cut into `split` narrower items (1, 2 or 4)
    int items;            // full_items + (tiles - full_items) * split
};

// Work item j (CTA j % grid takes it): output rows [n0, n0 + 128) x activation rows
// [m0, m0 + width). Whole tiles fill the complete rounds of the grid; the tiles of the
// last, partial round are cut along the activation rows so that round is shorter.
struct Item {
    int n0, m0, width;
};
Q4_DEVINL Item item_of(const PrefillArgs &a, int j) {
    Item it;
    int t = j, part = 0;
    it.width = kBN;
    if (j >= a.full_items) {
        t = a.full_items + (j - a.full_items) / a.split;
        part = (j - a.full_items) % a.split;
        it.width = kBN / a.split;
    }
    it.n0 = (t % a.tiles_n) * kBM;
    it.m0 = (t / a.tiles_n) * kBN + part * it.width;
    return it;
}

// ---- tcgen05 helpers -------------------------------------------------------------------
Q4_DEVINL void tmem_alloc(uint32_t *dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)),
                 "r"(ncols)
                 : "memory");
}
Q4_DEVINL void tmem_relinquish() { asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory"); }
Q4_DEVINL void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
Q4_DEVINL void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
Q4_DEVINL void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
// D[tmem] (+)= A[smem desc] * B[smem desc]^T, kind::f16 (bf16 in, fp32 accumulate)
Q4_DEVINL void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// Arrive once on `bar` when every tcgen05 operation issued so far by this thread is done.
Q4_DEVINL void umma_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}
Q4_DEVINL void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
}
// acc (a pair of fp32 in one 64-bit register) += s2 * (lo, hi), one packed instruction.
Q4_DEVINL void fma2_acc(uint64_t &acc, uint64_t s2, uint32_t lo, uint32_t hi) {
    asm("{\n\t.reg .b64 v;\n\tmov.b64 v, {%1, %2};\n\tfma.rn.f32x2 %0, %3, v, %0;\n\t}"
        : "+l"(acc)
        : "r"(lo), "r"(hi), "l"(s2));
}
Q4_DEVINL void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
// Generic-proxy shared-memory writes become visible to the tensor core (async proxy).
Q4_DEVINL void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, rows of 128 bytes, 8-row
// groups 1024 bytes apart (the layout a 128-byte-swizzle TMA writes).
Q4_DEVINL uint64_t sw128_desc(const void *p) {
    const uint32_t a = smem_u32(p);
    uint64_t d = (uint64_t)((a >> 4) & 0x3FFF);
    d |= (uint64_t)1 << 16;             // leading byte offset (unused with swizzle): 16 B
    d |= (uint64_t)(1024 >> 4) << 32;   // stride byte offset: 1024 B between 8-row groups
    d |= (uint64_t)1 << 46;             // descriptor version (sm_100)
    d |= (uint64_t)2 << 61;             // SWIZZLE_128B
    return d;
}
// Instruction descriptor: D fp32, A and B bf16, both K-major, N = 256, M = 128.
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kBN >> 3) << 17) |
                            ((uint32_t)(kBM >> 4) << 24);

Q4_DEVINL uint32_t bsub2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
Q4_DEVINL uint32_t pack_bf16x2(float lo, float hi) {
    uint32_t d;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
    return d;
}

// 8 codes of a 32-bit int4 word (k ascending: byte j holds k 2j in its low nibble) as 8
// bf16 in k order: (0x4300 | u) is the bf16 128 + u; minus 136 is u - 8 = code (exact).
Q4_DEVINL uint4 codes_int4(uint32_t w) {
    const uint32_t w4 = w >> 4;
    uint32_t r[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint32_t sel = (uint32_t)(j | (j << 4) | ((4 + j) << 8) | ((4 + j) << 12));
        r[j] = bsub2((prmt(w, w4, sel) & 0x000F000Fu) | 0x43004300u, 0x43084308u);
    }
    return make_uint4(r[0], r[1], r[2], r[3]);
}
// 4 int8 codes (two's complement bytes, k ascending) as 4 bf16: the fp32 2^23 + (c + 128)
// is assembled from the byte, minus 2^23 + 128 is c (exact), then packed to bf16 (exact).
Q4_DEVINL uint2 codes_int8(uint32_t w) {
    const uint32_t v = w ^ 0x80808080u;
    float c[4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
        c[j] = __uint_as_float(prmt(v, 0x4B000000u, (uint32_t)(j | (5 << 4) | (5 << 8) | (7 << 12)))) - 8388736.0f;
    return make_uint2(pack_bf16x2(c[0], c[1]), pack_bf16x2(c[2], c[3]));
}

// PC: one scale group per tile (per-output-channel scales): the scale is applied once when
// the tile ends, so the epilogue keeps no accumulators and four epilogue warps suffice;
// the freed warps dequantize (int8 -> bf16 is the costlier conversion).
template <int BITS, bool PC>
__global__ void __launch_bounds__(PC ? kThreadsPC : kThreads, 1)
prefill_gemm(const PrefillArgs a, const __grid_constant__ CUtensorMap tmx, const __grid_constant__ CUtensorMap tmp) {
    constexpr int PB = kBM * kBK * BITS / 8;  // payload bytes per k-step (4 or 8 KB)
    constexpr int PROW = kBK * BITS / 8;      // payload bytes per row per k-step (32 or 64)
    constexpr int NDQW = PC ? 8 : 4;          // dequantizing warps (warps 2 .. 1 + NDQW)
    constexpr int NCH = PROW / 16;            // 16-byte payload chunks per row and k-step
    constexpr int UPT = kBM * NCH / (32 * NDQW);  // payload chunks per dequantizing thread
    constexpr int NEPW = PC ? 4 : 8;          // epilogue warps (the rest)
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint8_t *xs = smem;                                   // kStages x 32 KB
    uint8_t *as = xs + kStages * kXBytes;                 // kAStages x 16 KB
    uint8_t *ps = as + kAStages * kABytes;                // kStages x PB
    uint64_t *full = reinterpret_cast<uint64_t *>(ps + kStages * kPBytesMax);
    uint64_t *empty = full + kStages;
    uint64_t *afull = empty + kStages;
    uint64_t *aempty = afull + kAStages;
    uint64_t *dfull = aempty + kAStages;
    uint64_t *dempty = dfull + 2;
    uint64_t *done = dempty + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(done + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(full + i, 1);
            mbar_init(empty + i, 1 + NDQW);  // MMA commit + dequantizing warps
        }
        for (int i = 0; i < kAStages; ++i) {
            mbar_init(afull + i, NDQW);
            mbar_init(aempty + i, 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(dfull + i, 1);
            mbar_init(dempty + i, NEPW);
        }
        mbar_init(done, 1);
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    bool timed_out = false;
    const int ntile_cta = a.items > (int)blockIdx.x ? (a.items - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;

    auto tma_role = [&]() {
        // ---------------- TMA producer ----------------
        if (lane == 0) {
            int it = 0;
            for (int tl = 0; tl < ntile_cta; ++tl) {
                const Item itm = item_of(a, blockIdx.x + tl * gridDim.x);
                const int n0 = itm.n0, m0 = itm.m0;
                for (int ks = 0; ks < a.ksteps; ++ks, ++it) {
                    const int s = it % kStages;
                    if (it >= kStages && !timed_out)
                        timed_out = !mbar_wait(empty + s, (uint32_t)(((it / kStages) - 1) & 1));
                    if (timed_out) break;
                    mbar_arrive_expect_tx(full + s, kXBytes + PB);
                    tma_load_2d(xs + s * kXBytes, &tmx, full + s, ks * kBK, m0);
                    tma_load_2d(ps + s * kPBytesMax, &tmp, full + s, ks * PROW, n0);
                }
                if (timed_out) break;
            }
        }
    };
    auto mma_role = [&]() {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            int it = 0, ait = 0, grp = 0;
            for (int tl = 0; tl < ntile_cta && !timed_out; ++tl) {
                const Item itm = item_of(a, blockIdx.x + tl * gridDim.x);
                const uint32_t idesc = (kIdesc & ~(0x3Fu << 17)) | ((uint32_t)(itm.width >> 3) << 17);
                for (int ks = 0; ks < a.ksteps; ++ks, ++it, ++ait) {
                    const int s = it % kStages, sa = ait % kAStages;
                    const int kg = ks % a.kpg, d = grp & 1;
                    if (kg == 0 && grp >= 2 && !timed_out)
                        timed_out = !mbar_wait(dempty + d, (uint32_t)(((grp >> 1) - 1) & 1));
                    if (!timed_out) timed_out = !mbar_wait(full + s, (uint32_t)((it / kStages) & 1));
                    if (!timed_out) timed_out = !mbar_wait(afull + sa, (uint32_t)((ait / kAStages) & 1));
                    if (timed_out) break;
                    tc_fence_after();
                    const uint32_t dt = tmem + (uint32_t)(d * kBN);
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk) {
                        umma_bf16(dt, sw128_desc(as + sa * kABytes + kk * 32), sw128_desc(xs + s * kXBytes + kk * 32),
                                  idesc, (kg > 0 || kk > 0) ? 1u : 0u);
                    }
                    umma_commit(empty + s);
                    umma_commit(aempty + sa);
                    if (kg == a.kpg - 1) {
                        umma_commit(dfull + d);
                        ++grp;
                    }
                }
            }
            umma_commit(done);
        }
    };
    auto dequant_role = [&]() {
        // ---------------- dequantize: payload -> bf16 codes (A) ----------------
        const int dt = threadIdx.x - 64;  // payload chunks dt + 32 * NDQW * i, i < UPT
        int it = 0, ait = 0;
        for (int tl = 0; tl < ntile_cta && !timed_out; ++tl) {
            for (int ks = 0; ks < a.ksteps; ++ks, ++it, ++ait) {
                const int s = it % kStages, sa = ait % kAStages;
                if (!timed_out) timed_out = !mbar_wait(full + s, (uint32_t)((it / kStages) & 1));
                if (ait >= kAStages && !timed_out)
                    timed_out = !mbar_wait(aempty + sa, (uint32_t)(((ait / kAStages) - 1) & 1));
                if (timed_out) break;
                const uint8_t *pst = ps + s * kPBytesMax;
                uint8_t *ast = as + sa * kABytes;
                if constexpr (PC) {
                    // consecutive threads take consecutive 16-byte payload chunks (conflict-free
                    // reads); chunk c of row r becomes 4 (int4) or 2 (int8) 16-byte chunks of
                    // the swizzled A row, which 8 neighbouring threads spread over all banks
    #pragma unroll
                    for (int i = 0; i < UPT; ++i) {
                        const int u = dt + 32 * NDQW * i;
                        const int r = u / NCH, c = u % NCH;
                        const uint4 p = *reinterpret_cast<const uint4 *>(pst + r * PROW + 16 * c);
                        const uint32_t wd[4] = {p.x, p.y, p.z, p.w};
                        uint8_t *dst = ast + r * 128;
                        if constexpr (BITS == 4) {
    #pragma unroll
                            for (int q = 0; q < 4; ++q)
                                *reinterpret_cast<uint4 *>(dst + (((4 * c + q) ^ (r & 7)) << 4)) = codes_int4(wd[q]);
                        } else {
    #pragma unroll
                            for (int q = 0; q < 2; ++q) {
                                const uint2 lo = codes_int8(wd[2 * q]), hi = codes_int8(wd[2 * q + 1]);
                                *reinterpret_cast<uint4 *>(dst + (((2 * c + q) ^ (r & 7)) << 4)) =
                                    make_uint4(lo.x, lo.y, hi.x, hi.y);
                            }
                        }
                    }
                } else {
                    // whole rows: row dt (and dt + 32 * NDQW, ... while rows remain)
#pragma unroll
                    for (int h = 0; h < kBM / (32 * NDQW); ++h) {
                        const int r = dt + 32 * NDQW * h;
                        const uint4 *src = reinterpret_cast<const uint4 *>(pst + r * PROW);
                        uint8_t *dst = ast + r * 128;
                        // rows sit 32 (int4) or 64 (int8) bytes apart, so the lanes of one
                        // shared-memory phase would read the same banks; each lane starts at a
                        // chunk that depends on its row, which spreads them over all banks
                        if constexpr (BITS == 4) {
                            const int j0 = (r >> 2) & 1;  // rows r and r + 4 take different halves first
                            const uint4 pa = src[j0], pb = src[j0 ^ 1];
                            const uint4 p0 = j0 ? pb : pa, p1 = j0 ? pa : pb;  // 64 codes
                            const uint32_t wds[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
#pragma unroll
                            for (int c = 0; c < 8; ++c)
                                *reinterpret_cast<uint4 *>(dst + ((c ^ (r & 7)) << 4)) = codes_int4(wds[c]);
                        } else {
#pragma unroll
                            for (int c0 = 0; c0 < 8; ++c0) {
                                const int c = (c0 + r) & 7;
                                const uint2 wv = reinterpret_cast<const uint2 *>(src)[c];  // 8 codes
                                const uint2 lo = codes_int8(wv.x), hi = codes_int8(wv.y);
                                *reinterpret_cast<uint4 *>(dst + ((c ^ (r & 7)) << 4)) =
                                    make_uint4(lo.x, lo.y, hi.x, hi.y);
                            }
                        }
                    }
                }
                fence_async_smem();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(afull + sa);
                    mbar_arrive(empty + s);
                }
            }
        }
    };
    auto epilogue_pc = [&]() {
        // ---------------- epilogue, one group per tile: y = scale * D ----------------
        const int q = warp & 3;
        const int rl = 32 * q + lane;
        const uint32_t lane_base = tmem + ((uint32_t)(32 * q) << 16);
        for (int tl = 0; tl < ntile_cta && !timed_out; ++tl) {
            const Item itm = item_of(a, blockIdx.x + tl * gridDim.x);
            const int n = itm.n0 + rl, d = tl & 1;
            const float sc = a.scales[min(n, a.N - 1)];
            timed_out = !mbar_wait(dfull + d, (uint32_t)((tl >> 1) & 1));
            if (timed_out) break;
            tc_fence_after();
            for (int ch = 0; ch < kBN / 32; ++ch) {
                if (32 * ch >= itm.width) break;
                uint32_t v0[16], v1[16];
                tmem_ld16(lane_base + (uint32_t)(d * kBN + 32 * ch), v0);
                tmem_ld16(lane_base + (uint32_t)(d * kBN + 32 * ch + 16), v1);
                tmem_wait_ld();
                if (n < a.N) {
                    const int mb = itm.m0 + 32 * ch, lim = min(itm.width - 32 * ch, a.M - mb);
                    float *yp = a.y + (size_t)mb * a.N + n;
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        if (i < lim) yp[(size_t)i * a.N] = sc * __uint_as_float(v0[i]);
                        if (16 + i < lim) yp[(size_t)(16 + i) * a.N] = sc * __uint_as_float(v1[i]);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(dempty + d);
        }
    };
    auto epilogue_grouped = [&]() {
        // ---------------- epilogue: promotion and stores ----------------
        const int q = warp & 3, half = (warp - 8) >> 2;
        const int rl = 32 * q + lane;                       // weight row inside the tile
        const uint32_t lane_base = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(128 * half);
        int grp = 0;
        for (int tl = 0; tl < ntile_cta && !timed_out; ++tl) {
            const Item itm = item_of(a, blockIdx.x + tl * gridDim.x);
            const int n0 = itm.n0, m0 = itm.m0;
            const int ncols = min(max(itm.width - 128 * half, 0), 128);  // this warp's valid columns
            const int n = n0 + rl;
            const float *srow = a.scales + (size_t)min(n, a.N - 1) * a.scales_per_row;
            uint64_t acc[64];  // 128 fp32 accumulators, two per register pair
#pragma unroll
            for (int i = 0; i < 64; ++i) acc[i] = 0ull;
            const int ngroups = a.ksteps / a.kpg;
            float s_next = srow[0];
            for (int gi = 0; gi < ngroups; ++gi, ++grp) {
                const int d = grp & 1;
                const float sc = s_next;
                const uint64_t s2 = ((uint64_t)__float_as_uint(sc) << 32) | __float_as_uint(sc);
                if (gi + 1 < ngroups) s_next = srow[gi + 1];
                if (!timed_out) timed_out = !mbar_wait(dfull + d, (uint32_t)((grp >> 1) & 1));
                if (timed_out) break;
                tc_fence_after();
#pragma unroll
                for (int ch = 0; ch < 4; ++ch) {
                    if (32 * ch >= ncols) break;  // narrow item: no more columns here
                    uint32_t v0[16], v1[16];      // two loads in flight per wait
                    tmem_ld16(lane_base + (uint32_t)(d * kBN + 32 * ch), v0);
                    tmem_ld16(lane_base + (uint32_t)(d * kBN + 32 * ch + 16), v1);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        fma2_acc(acc[16 * ch + i], s2, v0[2 * i], v0[2 * i + 1]);
                        fma2_acc(acc[16 * ch + 8 + i], s2, v1[2 * i], v1[2 * i + 1]);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(dempty + d);
            }
            if (timed_out) break;
            if (n < a.N) {
#pragma unroll
                for (int i = 0; i < 128; ++i) {
                    const int m = m0 + 128 * half + i;
                    const uint32_t bits = (i & 1) ? (uint32_t)(acc[i >> 1] >> 32) : (uint32_t)acc[i >> 1];
                    if (i < ncols && m < a.M) a.y[(size_t)m * a.N + n] = __uint_as_float(bits);
                }
            }
        }
    };
    if constexpr (PC) {
        if (warp == 0)
            tma_role();
        else if (warp == 1)
            mma_role();
        else if (warp < 2 + NDQW)
            dequant_role();
        else
            epilogue_pc();
    } else if (warp < 8) {
        // the first two warpgroups give registers up, at one program point for all 8 warps
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsLow));
        if (warp == 0)
            tma_role();
        else if (warp == 1)
            mma_role();
        else if (warp < 2 + NDQW)
            dequant_role();
        // warps 6 and 7: no role
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsHigh));
        epilogue_grouped();
    }


    // wait for the last MMAs before releasing tensor memory
    if (warp == 1 && lane == 0 && !timed_out) timed_out = !mbar_wait(done, 0);
    if (timed_out && a.status) atomicOr(a.status, Q4_STATUS_TIMEOUT);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

constexpr size_t smem_bytes() {
    return 1024 + (size_t)kStages * kXBytes + (size_t)kAStages * kABytes + (size_t)kStages * kPBytesMax +
           (2 * kStages + 2 * kAStages + 5) * 8 + 16;
}

}  // namespace

bool prefill_supported(int64_t M, int64_t N, int64_t K, int bits, int64_t group, bool x_bf16) {
    return x_bf16 && M >= 64 && K % kBK == 0 && group % kBK == 0 && K % group == 0 && N >= 1 &&
           K <= ((int64_t)1 << 30) && N <= ((int64_t)1 << 30) && M <= ((int64_t)1 << 30) && (bits == 4 || bits == 8);
}

cudaError_t launch_prefill(const void *x, int64_t M, const uint8_t *payload, const float *scales, int64_t N,
                           int64_t K, int bits, int64_t group, float *y, uint32_t *status, int sms,
                           cudaStream_t st) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return cudaErrorNotSupported;
    CUtensorMap tmx, tmp;
    {
        const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)M};
        const cuuint64_t strides[1] = {(cuuint64_t)K * 2};
        const cuuint32_t box[2] = {(cuuint32_t)kBK, (cuuint32_t)kBN};
        const cuuint32_t es[2] = {1, 1};
        if (enc(&tmx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(x), dims, strides, box, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    {
        const uint64_t rowbytes = (uint64_t)K * bits / 8;
        const cuuint64_t dims[2] = {rowbytes, (cuuint64_t)N};
        const cuuint64_t strides[1] = {rowbytes};
        const cuuint32_t box[2] = {(cuuint32_t)(kBK * bits / 8), (cuuint32_t)kBM};
        const cuuint32_t es[2] = {1, 1};
        if (enc(&tmp, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(payload), dims, strides, box, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    PrefillArgs a;
    a.scales = scales;
    a.y = y;
    a.status = status;
    a.M = (int)M;
    a.N = (int)N;
    a.K = (int)K;
    a.scales_per_row = (int)(K / group);
    a.kpg = (int)(group / kBK);
    a.ksteps = (int)(K / kBK);
    a.tiles_n = (int)((N + kBM - 1) / kBM);
    a.tiles = a.tiles_n * (int)((M + kBN - 1) / kBN);
    const int grid = a.tiles < sms ? a.tiles : sms;
    // complete rounds of whole tiles; the last partial round is cut in 2 or 4 along the
    // activation rows when the pieces still fit in one round
    a.full_items = a.tiles / grid * grid;
    const int rem = a.tiles - a.full_items;
    a.split = rem == 0 ? 1 : rem * 4 <= grid ? 4 : rem * 2 <= grid ? 2 : 1;
    a.items = a.full_items + rem * a.split;
    const size_t smem = smem_bytes();
    const bool pc = a.kpg == a.ksteps;  // one scale group per tile
    auto kern = bits == 4 ? (pc ? prefill_gemm<4, true> : prefill_gemm<4, false>)
                          : (pc ? prefill_gemm<8, true> : prefill_gemm<8, false>);
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    if (!pc) {
        // the register split above assumes the block launches at exactly kRegsLaunch a
        // thread; any other allocation could leave an increase waiting: refuse to launch
        static int regs[2] = {0, 0};
        int &rg = regs[bits == 4 ? 0 : 1];
        if (!rg) {
            cudaFuncAttributes fa;
            const cudaError_t ae = cudaFuncGetAttributes(&fa, kern);
            if (ae != cudaSuccess) return ae;
            rg = fa.numRegs;
        }
        if (rg != kRegsLaunch) return cudaErrorInvalidConfiguration;
    }
    kern<<<grid, pc ? kThreadsPC : kThreads, smem, st>>>(a, tmx, tmp);
    return cudaGetLastError();
}

}  // namespace q4
