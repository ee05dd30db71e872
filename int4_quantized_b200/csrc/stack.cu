// stack.cu -- the decode GEMVs of a whole model step in one persistent kernel.
//
// "Huit bits, puis quatre", section "La vitesse": a decode step that launches one short
// kernel per layer spends its time in launches and pipeline fills, not in reading the
// weights; the page expects the quantized weights to pay off only once the kernels are
// fused so that they really wait on memory. This kernel runs every GEMV of a step (one
// row of x each, the qgemm arithmetic of gemv_math.cuh) in one launch:
//
//   * GEMVs are grouped in levels. The GEMVs of a level read activations that are ready
//     when the level starts (the outputs of earlier levels, or inputs given by the
//     caller); level l + 1 may read what level l writes (q/k/v, then o, then gate/up,
//     then down, in a transformer layer).
//   * The weight tiles (128 rows x 128 bytes) of a level are numbered GEMV by GEMV, row
//     block by row block, k-stage by k-stage, and each of the G resident CTAs takes one
//     contiguous G-th of them (an even split of the level's bytes, whatever its shapes).
//   * A producer warp per CTA streams the CTA's tiles of every level, in order, through
//     one TMA ring, with the scales of each tile beside it. It never waits for a level:
//     the weights are static, so the next level's tiles arrive while the current level
//     ends and its activations are published.
//   * Eight consumer warps wait (bounded, on a device counter) until the previous level
//     is complete, build the bf16 pieces of x for their tiles, and multiply. A row block
//     whose k-stages were split over several CTAs is added up by whichever CTA finishes
//     its share last, from the partial sums in fixed CTA order (deterministic results).
//     A completed row block increments the level's counter.
//   * Counters return to zero at the end of every launch (the last CTA to finish resets
//     them), so the workspace can be replayed, e.g. from a CUDA graph.
//
// Every wait is bounded (about one second); one that gives up sets Q4_STATUS_TIMEOUT and
// the CTA goes on without waiting, so the launch always ends. Before a CTA exits, its
// producer waits (bounded) for every copy it issued into the CTA's shared memory.
#include <cuda.h>

#include <cstring>
#include <vector>

#include "common.cuh"
#include "gemv_math.cuh"
#include "kernels.h"

namespace q4 {

namespace {

using namespace gm;

constexpr int kConsumers = 8;
constexpr int kConsumerThreads = 32 * kConsumers;
constexpr int kThreads = kConsumerThreads + 32;
constexpr int kRing = 5;                   // payload stages in flight per CTA
constexpr int kSmemBudget = 115200;        // two CTAs per SM
constexpr int kCtasPerSm = 2;

struct alignas(64) StackEntry {
    CUtensorMap tm;        // 2D map of the payload: {row bytes, N}, box 128 x 128, 128B swizzle
    const float *scales;
    const void *x;
    float *y;
    int64_t unit_base;     // first tile of this GEMV in its level's numbering
    int N, K;
    int group;             // scale group (divides K)
    int spr;               // scales per row = K / group
    int S;                 // k-stages per row (128 bytes of payload each)
    int R;                 // row blocks of 128
    int task_base;         // global index of row block 0
    int level;
};

struct StackLevel {
    int64_t U;             // tiles in the level
    int e0, ne;            // its GEMVs
    int T;                 // row blocks in the level
    int pad;
};

struct StackArgs {
    const StackEntry *ent;
    const StackLevel *lev;
    int *task_cnt;         // [n_tasks] arrivals of the CTAs sharing a row block
    int *level_done;       // [L] completed row blocks per level
    int *finished;         // CTAs done with the launch
    int *tflag;            // set when a wait gave up: the last CTA also resets task_cnt
    float *partial;        // [G][2][128] partial sums
    uint32_t *status;
    int G, L, n_tasks;
    int P;                 // pieces per activation: 3 (fp32 x) or 1 (bf16 x)
    int ucap;              // tiles whose activation pieces fit in shared memory at once
    int gs;                // scale slots per row per tile (max(1, groups per tile))
    uint64_t wait_ns;      // bound of every wait
};

Q4_DEVINL int ld_acquire(const int *p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
Q4_DEVINL float ld_cg_f32(const float *p) {
    float v;
    asm volatile("ld.global.cg.f32 %0, [%1];" : "=f"(v) : "l"(p) : "memory");
    return v;
}
Q4_DEVINL void tmap_acquire(const CUtensorMap *tm) {
    asm volatile("fence.proxy.tensormap::generic.acquire.gpu [%0], 128;" ::"l"(tm) : "memory");
}
Q4_DEVINL void tma_load_2d_g(void *dst, const CUtensorMap *tmap, uint64_t *bar, int c0, int c1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];"
        ::"r"(smem_u32(dst)), "l"(tmap), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
        : "memory");
}

// Tiles [u0, u1) of a level with U tiles that CTA c of G owns.
Q4_DEVINL void cta_range(int64_t U, int c, int G, int64_t &u0, int64_t &u1) {
    u0 = U * c / G;
    u1 = U * (c + 1) / G;
}
// The CTA that owns tile u of a level with U tiles.
Q4_DEVINL int cta_of(int64_t u, int64_t U, int G) { return (int)(((u + 1) * G - 1) / U); }

// Entry of tile u (level-local), searching forward from e.
Q4_DEVINL int locate(const StackEntry *ent, int e, int e_end, int64_t u) {
    while (e + 1 < e_end && u >= ent[e + 1].unit_base) ++e;
    return e;
}

Q4_DEVINL bool wait_counter(const int *p, int target, uint64_t limit_ns) {
    if (ld_acquire(p) >= target) return true;
    const uint64_t t0 = global_ns();
    for (;;) {
        __nanosleep(64);
        if (ld_acquire(p) >= target) return true;
        if (global_ns() - t0 > limit_ns) return false;
    }
}

template <int BITS, int L, int GPS, bool XBF16>
__global__ void __maxnreg__(96) gemv_stack(const StackArgs a) {
    constexpr int SPS = kTileBytes / (4 * L);
    constexpr int KTI = BITS == 4 ? L / 2 : L / 4;
    constexpr int KTS = SPS * KTI;
    constexpr int WPT = L / 4;
    constexpr int STAGEK = kTileBytes * 8 / BITS;
    constexpr int GS = GPS > 0 ? GPS : 1;
    constexpr int FSLOT = KTS * 16 * 8;  // piece bytes of one tile (16 lanes stored)
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint8_t *ring = smem;                                                  // kRing x 16 KB
    float *scl = reinterpret_cast<float *>(ring + kRing * kTileWords);    // kRing x [128][GS]
    float *redc = scl + kRing * kTileRows * GS;                           // [128][8]
    uint8_t *bbuf = reinterpret_cast<uint8_t *>(redc + kTileRows * 8);     // ucap x FSLOT
    uint64_t *full = reinterpret_cast<uint64_t *>(bbuf + (size_t)a.ucap * FSLOT);
    uint64_t *empty = full + kRing;
    int *flag = reinterpret_cast<int *>(empty + kRing);  // [0]: last arriver, [1]: timed out

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int c = blockIdx.x, G = a.G;
    if (threadIdx.x == 0) {
        for (int i = 0; i < kRing; ++i) {
            mbar_init(full + i, 1 + 32);  // the TMA's expect_tx arrival + 32 lanes' scale copies
            mbar_init(empty + i, kConsumers);
        }
        flag[0] = flag[1] = 0;
        fence_barrier_init();
    }
    __syncthreads();
    bool timed_out = false;

    if (warp == kConsumers) {
        // ---------------- producer warp: every tile of every level, in order ----------------
        int slot = 0, round = 0;
        int issued[kRing];
#pragma unroll
        for (int i = 0; i < kRing; ++i) issued[i] = 0;
        for (int l = 0; l < a.L; ++l) {
            const StackLevel lv = a.lev[l];
            int64_t u0, u1;
            cta_range(lv.U, c, G, u0, u1);
            int e = lv.e0;
            int e_acq = -1;
            for (int64_t u = u0; u < u1; ++u) {
                e = locate(a.ent, e, lv.e0 + lv.ne, u);
                const StackEntry &E = a.ent[e];
                if (e != e_acq) {
                    tmap_acquire(&E.tm);
                    e_acq = e;
                }
                const int64_t ul = u - E.unit_base;
                const int rb = (int)(ul / E.S), s = (int)(ul - (int64_t)rb * E.S);
                if (round > 0 && !timed_out) timed_out = !mbar_wait(empty + slot, (uint32_t)((round - 1) & 1), a.wait_ns);
                if (lane == 0 && !timed_out) {
                    mbar_arrive_expect_tx(full + slot, kTileWords);
                    tma_load_2d_g(ring + slot * kTileWords, &E.tm, full + slot, s * kTileBytes, rb * kTileRows);
                }
                // the tile's scales: GS per row (the groups of the stage), clamped to the row
                const int gbase = GPS > 0 ? s * GPS : (s * STAGEK) / E.group;
                const int ng = min(GS, E.spr - gbase);
                float *dst = scl + slot * kTileRows * GS;
                for (int r = lane; r < kTileRows; r += 32) {
                    const int n = min(rb * kTileRows + r, E.N - 1);
                    const float *src = E.scales + (size_t)n * E.spr + gbase;
                    for (int q = 0; q < ng; ++q) cp_async4(dst + r * GS + q, src + q);
                }
                cp_async_arrive(full + slot);
                ++issued[slot];
                if (++slot == kRing) { slot = 0; ++round; }
            }
        }
        // drain: every copy issued into this CTA's shared memory has landed before it exits
#pragma unroll
        for (int i = 0; i < kRing; ++i)
            if (issued[i] > 0) (void)mbar_wait(full + i, (uint32_t)((issued[i] - 1) & 1), a.wait_ns);
    } else {
        // ---------------- consumers ----------------
        const int g = lane >> 2, t = lane & 3;
        const int ct = threadIdx.x;
        const int pr = 16 * warp + row_perm<L>(g);
        uint32_t aoff[SPS];
#pragma unroll
        for (int sl = 0; sl < SPS; ++sl) {
            const int off = sl * 4 * L + t * L;
            aoff[sl] = pr * kTileBytes + (((off >> 4) ^ (pr & 7)) << 4) + (off & 15);
        }
        const int fl = lane & 15;
        float acc[1][4] = {{0.f, 0.f, 0.f, 0.f}};
        int slot = 0, round = 0;
        for (int l = 0; l < a.L; ++l) {
            const StackLevel lv = a.lev[l];
            int64_t u0, u1;
            cta_range(lv.U, c, G, u0, u1);
            if (u0 == u1) continue;
            if (l > 0) {
                // the activations of this level are complete once every row block of the
                // previous level is
                if (ct == 0 && !timed_out) {
                    timed_out = !wait_counter(a.level_done + (l - 1), a.lev[l - 1].T, a.wait_ns);
                    __threadfence();
                }
                named_barrier_sync(1, kConsumerThreads);
            }
            int e = locate(a.ent, lv.e0, lv.e0 + lv.ne, u0);
            int64_t chunk_end = u0;
            for (int64_t u = u0; u < u1; ++u) {
                if (u == chunk_end) {
                    // pieces of x for the next ucap tiles (every warp is done with the last ones)
                    if (u != u0) named_barrier_sync(1, kConsumerThreads);
                    chunk_end = min(u1, u + a.ucap);
                    constexpr int IPT = STAGEK / 8;  // 8-k items per tile
                    const int items = (int)(chunk_end - u) * IPT;
                    int ei = e;
                    for (int it = ct; it < items; it += kConsumerThreads) {
                        const int j = it / IPT, kk = 8 * (it - j * IPT);
                        const int64_t uu = u + j;
                        ei = locate(a.ent, e, lv.e0 + lv.ne, uu);
                        const StackEntry &E = a.ent[ei];
                        const int s = (int)((uu - E.unit_base) % E.S);
                        const int k = s * STAGEK + kk;
                        float v[8];
                        if (k < E.K) {
                            load_x8<XBF16, true>(E.x, k, v);
                        } else {
#pragma unroll
                            for (int q = 0; q < 8; ++q) v[q] = 0.f;
                        }
                        float z[8];
#pragma unroll
                        for (int q = 0; q < 8; ++q) z[q] = 0.f;
                        uint2 *st = reinterpret_cast<uint2 *>(bbuf + (size_t)j * FSLOT);
                        frag_unit<BITS, L>(st, kk, 0, v, a.P, 4, 1, 16, true);
                        for (int vm = 1; vm * a.P < 4; ++vm) frag_unit<BITS, L>(st, kk, vm, z, a.P, 4, 1, 16, true);
                    }
                    named_barrier_sync(1, kConsumerThreads);
                }
                e = locate(a.ent, e, lv.e0 + lv.ne, u);
                const StackEntry &E = a.ent[e];
                const int64_t ul = u - E.unit_base;
                const int rb = (int)(ul / E.S), s = (int)(ul - (int64_t)rb * E.S);
                const int seg_hi = (E.K * BITS / 8) / (4 * L);  // segments per row
                const int nsl = min(SPS, seg_hi - s * SPS);
                if (!timed_out) timed_out = !mbar_wait(full + slot, (uint32_t)(round & 1), a.wait_ns);
                const uint8_t *stg = ring + slot * kTileWords;
                uint32_t A0[SPS][WPT], A1[SPS][WPT];
#pragma unroll
                for (int sl = 0; sl < SPS; ++sl) {
                    lds_words<L>(A0[sl], stg + aoff[sl]);
                    lds_words<L>(A1[sl], stg + aoff[sl] + 8 * kTileBytes);
                }
                float s0r[GS], s1r[GS];
                const float *sc = scl + slot * kTileRows * GS;
#pragma unroll
                for (int q = 0; q < GS; ++q) {
                    s0r[q] = sc[pr * GS + q];
                    s1r[q] = sc[(pr + 8) * GS + q];
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(empty + slot);  // codes and scales are in registers
                if (++slot == kRing) { slot = 0; ++round; }
                const int64_t cstart = u0 + ((u - u0) / a.ucap) * a.ucap;
                const uint8_t *fr = bbuf + (size_t)(u - cstart) * FSLOT + fl * 16;
                if (nsl == SPS)
                    stage_fixed<BITS, L, 1, 16, GPS, true>(A0, A1, fr, s0r, s1r, nsl, acc);
                else
                    stage_fixed<BITS, L, 1, 16, GPS, false>(A0, A1, fr, s0r, s1r, nsl, acc);

                // ---- end of this CTA's share of row block rb ----
                if (s == E.S - 1 || u == u1 - 1) {
                    const int T = E.task_base + rb;
                    const bool whole = (s == E.S - 1) && (u - s >= u0);  // every stage of the row block was here
                    __syncwarp();
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        redc[pr * 8 + 2 * t + q] = acc[0][q];
                        redc[(pr + 8) * 8 + 2 * t + q] = acc[0][2 + q];
                    }
                    __syncwarp();
                    if (lane < 16) {
                        const int r = 16 * warp + lane;
                        const float *src = redc + r * 8;
                        float v = src[0];
                        for (int p = 1; p < a.P; ++p) v += src[p];
                        if (whole) {
                            const int n = rb * kTileRows + r;
                            if (n < E.N) E.y[n] = v;
                        } else {
                            // which of this CTA's two partial slots: its first row block, or another
                            int ef = locate(a.ent, lv.e0, lv.e0 + lv.ne, u0);
                            const int Tf = a.ent[ef].task_base + (int)((u0 - a.ent[ef].unit_base) / a.ent[ef].S);
                            a.partial[((size_t)c * 2 + (T == Tf ? 0 : 1)) * kTileRows + r] = v;
                        }
                    }
#pragma unroll
                    for (int q = 0; q < 4; ++q) acc[0][q] = 0.f;
                    named_barrier_sync(1, kConsumerThreads);
                    const int64_t tf = E.unit_base + (int64_t)rb * E.S, tl = tf + E.S - 1;
                    const int cf = cta_of(tf, lv.U, G), clast = cta_of(tl, lv.U, G);
                    if (ct == 0) {
                        __threadfence();
                        if (whole) {
                            atomicAdd(a.level_done + l, 1);
                        } else {
                            int arrivals = 0;
                            for (int cc = cf; cc <= clast; ++cc) {
                                int64_t a0, a1;
                                cta_range(lv.U, cc, G, a0, a1);
                                arrivals += a0 < a1;
                            }
                            const int old = atomicAdd(a.task_cnt + T, 1);
                            flag[0] = old == arrivals - 1;
                        }
                    }
                    if (!whole) {
                        named_barrier_sync(1, kConsumerThreads);
                        if (flag[0]) {
                            // the last CTA of the row block adds the partial sums in CTA order
                            __threadfence();
                            if (ct < kTileRows) {
                                float v = 0.f;
                                bool first = true;
                                for (int cc = cf; cc <= clast; ++cc) {
                                    int64_t a0, a1;
                                    cta_range(lv.U, cc, G, a0, a1);
                                    if (a0 >= a1) continue;
                                    const int ec = locate(a.ent, lv.e0, lv.e0 + lv.ne, a0);
                                    const int Tc = a.ent[ec].task_base + (int)((a0 - a.ent[ec].unit_base) / a.ent[ec].S);
                                    const float pv = ld_cg_f32(a.partial + ((size_t)cc * 2 + (T == Tc ? 0 : 1)) * kTileRows + ct);
                                    v = first ? pv : v + pv;
                                    first = false;
                                }
                                const int n = rb * kTileRows + ct;
                                if (n < E.N) E.y[n] = v;
                            }
                            named_barrier_sync(1, kConsumerThreads);
                            if (ct == 0) {
                                a.task_cnt[T] = 0;
                                __threadfence();
                                atomicAdd(a.level_done + l, 1);
                            }
                        }
                    }
                }
            }
        }
    }
    if (timed_out) flag[1] = 1;
    __syncthreads();
    if (threadIdx.x == 0) {
        if (flag[1]) {
            if (a.status) atomicOr(a.status, Q4_STATUS_TIMEOUT);
            atomicExch(a.tflag, 1);
        }
        __threadfence();
        const int old = atomicAdd(a.finished, 1);
        if (old == G - 1) {
            // every CTA is done with the counters: return them to zero for the next launch
            __threadfence();
            for (int l = 0; l < a.L; ++l) a.level_done[l] = 0;
            if (atomicAdd(a.tflag, 0)) {
                for (int i = 0; i < a.n_tasks; ++i) a.task_cnt[i] = 0;
                *a.tflag = 0;
            }
            *a.finished = 0;
            __threadfence();
        }
    }
}

}  // namespace
}  // namespace q4

// ======================================================================================
// Host side: plan, prepare, run
// ======================================================================================
namespace q4 {
namespace {

constexpr int kPlanGrid = 148 * kCtasPerSm;  // partial-sum slots are sized for a full B200
constexpr uint64_t kPlanMagic = 0x71347374616b3031ull;

inline size_t al256(size_t v) { return (v + 255) / 256 * 256; }

// (L, groups per tile) of the GEMV for this format, as gemv_plan chooses them; false for
// groups the stack kernel does not cover (not dividing K, not a multiple of 32, or an
// irregular count per tile).
bool stack_format(int bits, int64_t K, int64_t group, int *L, int *gps) {
    if (K % 32 != 0 || group < 32 || K % group != 0 || group % 32 != 0) return false;
    if (bits == 4)
        *L = group % 128 == 0 ? 16 : group % 64 == 0 ? 8 : 4;
    else
        *L = group % 64 == 0 ? 16 : 8;
    const int64_t sk = kTileBytes * 8 / bits;
    int g = sk % group == 0 ? (int)(sk / group) : group % sk == 0 ? 0 : -1;
    if (g == 1) g = 0;
    if (g < 0) return false;
    *gps = g;
    return true;
}

struct StackLayout {
    int L, gps, nlev, n_tasks;
    size_t off_ent, off_lev, off_cnt, off_done, off_misc, off_part, bytes;
};

q4_status stack_layout(const q4_stack_gemv *gv, int32_t count, int bits, q4_xdtype xt, StackLayout *lo) {
    if (!gv || count < 1 || (bits != 4 && bits != 8) || (xt != Q4_X_F32 && xt != Q4_X_BF16)) return Q4_ERR_ARG;
    int64_t tasks = 0;
    for (int32_t i = 0; i < count; ++i) {
        const q4_stack_gemv &g = gv[i];
        if (!g.payload || !g.scales || !g.x || !g.y) return Q4_ERR_ARG;
        if (g.N < 1 || g.K < 1 || g.group < 1 || g.reserved != 0) return Q4_ERR_ARG;
        if (g.N > ((int64_t)1 << 30) || g.K > ((int64_t)1 << 30)) return Q4_ERR_UNSUPPORTED;
        if ((uintptr_t)g.payload % 16 || (uintptr_t)g.x % 16) return Q4_ERR_UNSUPPORTED;
        if (i == 0 ? g.level != 0 : (g.level != gv[i - 1].level && g.level != gv[i - 1].level + 1)) return Q4_ERR_ARG;
        int L, gps;
        if (!stack_format(bits, g.K, g.group, &L, &gps)) return Q4_ERR_UNSUPPORTED;
        if (i == 0) {
            lo->L = L;
            lo->gps = gps;
        } else if (L != lo->L || gps != lo->gps) {
            return Q4_ERR_UNSUPPORTED;  // one kernel variant per stack
        }
        tasks += (g.N + kTileRows - 1) / kTileRows;
    }
    if (tasks > (int64_t)1 << 30) return Q4_ERR_UNSUPPORTED;
    lo->nlev = gv[count - 1].level + 1;
    lo->n_tasks = (int)tasks;
    lo->off_ent = 0;
    lo->off_lev = al256((size_t)count * sizeof(StackEntry));
    lo->off_cnt = lo->off_lev + al256((size_t)lo->nlev * sizeof(StackLevel));
    lo->off_done = lo->off_cnt + al256((size_t)lo->n_tasks * 4);
    lo->off_misc = lo->off_done + al256((size_t)lo->nlev * 4);
    lo->off_part = lo->off_misc + 256;
    lo->bytes = lo->off_part + al256((size_t)kPlanGrid * 2 * kTileRows * 4);
    return Q4_OK;
}

using StackKernel = void (*)(StackArgs);

template <int BITS, int L, int GPS>
StackKernel pick(bool bf16) {
    return bf16 ? gemv_stack<BITS, L, GPS, true> : gemv_stack<BITS, L, GPS, false>;
}

StackKernel stack_kernel(int bits, int L, int gps, bool bf16) {
    if (bits == 4) {
        if (L == 16 && gps == 2) return pick<4, 16, 2>(bf16);
        if (L == 16 && gps == 0) return pick<4, 16, 0>(bf16);
        if (L == 8 && gps == 4) return pick<4, 8, 4>(bf16);
        if (L == 4 && gps == 8) return pick<4, 4, 8>(bf16);
    } else {
        if (L == 16 && gps == 2) return pick<8, 16, 2>(bf16);
        if (L == 16 && gps == 0) return pick<8, 16, 0>(bf16);
        if (L == 8 && gps == 4) return pick<8, 8, 4>(bf16);
    }
    return nullptr;
}

struct StackPlanImpl {
    uint64_t magic;
    StackKernel kern;
    StackArgs args;
    int grid;
    int pad;
    size_t smem;
};
static_assert(sizeof(StackPlanImpl) <= sizeof(q4_stack_plan), "plan fits the opaque struct");

}  // namespace
}  // namespace q4

extern "C" {

size_t q4_stack_workspace_bytes(const q4_stack_gemv *gemvs, int32_t count, int bits, q4_xdtype xt) {
    q4::StackLayout lo;
    if (q4::stack_layout(gemvs, count, bits, xt, &lo) != Q4_OK) return 0;
    return lo.bytes;
}

q4_status q4_stack_prepare(const q4_stack_gemv *gemvs, int32_t count, int bits, q4_xdtype xt, void *workspace,
                           size_t workspace_bytes, q4_stack_plan *plan, void *stream) {
    using namespace q4;
    if (!plan) return Q4_ERR_ARG;
    std::memset(plan, 0, sizeof *plan);
    StackLayout lo;
    q4_status st = stack_layout(gemvs, count, bits, xt, &lo);
    if (st != Q4_OK) return st;
    if (!workspace || (uintptr_t)workspace % 256 || workspace_bytes < lo.bytes) return Q4_ERR_WORKSPACE;
    if (!encode_fn()) return cuda_error(cudaErrorNotSupported, "cuTensorMapEncodeTiled");
    const bool bf16 = xt == Q4_X_BF16;
    StackKernel kern = stack_kernel(bits, lo.L, lo.gps, bf16);
    if (!kern) return Q4_ERR_UNSUPPORTED;

    // tables
    std::vector<StackEntry> ent(count);
    std::vector<StackLevel> lev(lo.nlev);
    int task_base = 0;
    for (int l = 0, i = 0; l < lo.nlev; ++l) {
        StackLevel &lv = lev[l];
        lv.e0 = i;
        lv.U = 0;
        lv.T = 0;
        lv.pad = 0;
        for (; i < count && gemvs[i].level == l; ++i) {
            const q4_stack_gemv &g = gemvs[i];
            StackEntry &E = ent[i];
            std::memset(&E, 0, sizeof E);
            if (!encode_payload_map(&E.tm, g.payload, g.N, g.K, bits)) return Q4_ERR_UNSUPPORTED;
            E.scales = g.scales;
            E.x = g.x;
            E.y = g.y;
            E.N = (int)g.N;
            E.K = (int)g.K;
            E.group = (int)g.group;
            E.spr = (int)(g.K / g.group);
            E.S = (int)((g.K * bits / 8 + kTileBytes - 1) / kTileBytes);
            E.R = (int)((g.N + kTileRows - 1) / kTileRows);
            E.task_base = task_base;
            E.level = l;
            E.unit_base = lv.U;
            lv.U += (int64_t)E.R * E.S;
            lv.T += E.R;
            task_base += E.R;
        }
        lv.ne = i - lv.e0;
    }

    // shared memory and grid
    const int stagek = kTileBytes * 8 / bits;
    const int kts = stagek / 16;
    const size_t fslot = (size_t)kts * 16 * 8;
    const int gsl = lo.gps > 0 ? lo.gps : 1;
    const size_t fixed = 1024 + (size_t)kRing * kTileWords + (size_t)kRing * kTileRows * gsl * 4 +
                         (size_t)kTileRows * 8 * 4 + 2 * kRing * 8 + 16;
    if (fixed + fslot > (size_t)kSmemBudget) return Q4_ERR_UNSUPPORTED;
    int ucap = (int)((kSmemBudget - fixed) / fslot);
    if (ucap > 64) ucap = 64;
    const size_t smem = fixed + (size_t)ucap * fslot;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return cuda_error(e, "stack kernel attribute");
    int dev = 0, sms = 0, per_sm = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return cuda_error(e, "cudaGetDevice");
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
        return cuda_error(e, "SM count");
    if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, smem)) != cudaSuccess)
        return cuda_error(e, "stack kernel occupancy");
    if (per_sm < 1) return Q4_ERR_UNSUPPORTED;
    int grid = sms * (per_sm < kCtasPerSm ? per_sm : kCtasPerSm);
    if (grid > kPlanGrid) grid = kPlanGrid;

    // copy the tables, zero the counters; the host tables can go once the stream is done
    char *w = static_cast<char *>(workspace);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if ((e = cudaMemcpyAsync(w + lo.off_ent, ent.data(), ent.size() * sizeof(StackEntry), cudaMemcpyHostToDevice,
                             s)) != cudaSuccess ||
        (e = cudaMemcpyAsync(w + lo.off_lev, lev.data(), lev.size() * sizeof(StackLevel), cudaMemcpyHostToDevice,
                             s)) != cudaSuccess ||
        (e = cudaMemsetAsync(w + lo.off_cnt, 0, lo.off_part - lo.off_cnt, s)) != cudaSuccess ||
        (e = cudaStreamSynchronize(s)) != cudaSuccess)
        return cuda_error(e, "stack tables");

    StackPlanImpl p = {};
    p.magic = kPlanMagic;
    p.kern = kern;
    p.args.ent = reinterpret_cast<const StackEntry *>(w + lo.off_ent);
    p.args.lev = reinterpret_cast<const StackLevel *>(w + lo.off_lev);
    p.args.task_cnt = reinterpret_cast<int *>(w + lo.off_cnt);
    p.args.level_done = reinterpret_cast<int *>(w + lo.off_done);
    p.args.finished = reinterpret_cast<int *>(w + lo.off_misc);
    p.args.tflag = reinterpret_cast<int *>(w + lo.off_misc) + 1;
    p.args.partial = reinterpret_cast<float *>(w + lo.off_part);
    p.args.status = nullptr;
    p.args.G = grid;
    p.args.L = lo.nlev;
    p.args.n_tasks = lo.n_tasks;
    p.args.P = bf16 ? 1 : 3;
    p.args.ucap = ucap;
    p.args.gs = gsl;
    p.args.wait_ns = kWaitLimitNs;
    p.grid = grid;
    p.smem = smem;
    std::memcpy(plan, &p, sizeof p);
    return Q4_OK;
}

q4_status q4_stack_set_wait_limit(q4_stack_plan *plan, uint64_t nanoseconds) {
    using namespace q4;
    if (!plan) return Q4_ERR_ARG;
    StackPlanImpl p;
    std::memcpy(&p, plan, sizeof p);
    if (p.magic != kPlanMagic) return Q4_ERR_ARG;
    p.args.wait_ns = nanoseconds;
    std::memcpy(plan, &p, sizeof p);
    return Q4_OK;
}

q4_status q4_stack_run(const q4_stack_plan *plan, uint32_t *status_word, void *stream) {
    using namespace q4;
    if (!plan) return Q4_ERR_ARG;
    StackPlanImpl p;
    std::memcpy(&p, plan, sizeof p);
    if (p.magic != kPlanMagic || !p.kern) return Q4_ERR_ARG;
    p.args.status = status_word;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = p.smem;
    cfg.stream = reinterpret_cast<cudaStream_t>(stream);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;  // every CTA resident at once: levels wait on each other
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cuda_error(cudaLaunchKernelEx(&cfg, p.kern, p.args), "stack launch");
}

}  // extern "C"
