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

// One CTA per SM: fifteen consumer warps (16 weight rows each) on 240-row tiles and one
// producer warp. Registers: 512 threads x 128 fill the SM's 64K; shared memory stays near
// 160 KB so that about 70 KB of the SM's 228 KB remain L1, which holds the lines of scales
// the consumers read (a 128-byte line serves a row over many consecutive stages).
constexpr int kConsumers = 15;
constexpr int kConsumerThreads = 32 * kConsumers;
constexpr int kThreads = kConsumerThreads + 32;
constexpr int kSRows = 16 * kConsumers;            // 240 weight rows per tile
constexpr int kSTile = kTileBytes * kSRows;        // 30 KB of codes per tile
constexpr int kRing = 4;                           // tiles in flight per CTA
constexpr int kSmemBudget = 163840;
constexpr int kCtasPerSm = 1;

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
    int *task_cnt;         // [n_tasks][15] arrivals of the CTAs sharing a row block, per warp
    int *level_done;       // [L] completed (row block, warp) pairs per level
    int *finished;         // CTAs done with the launch
    int *tflag;            // set when a wait gave up: the last CTA also resets task_cnt
    float *partial;        // [G][2][240] partial sums
    const int *ustart;     // [L][G + 1] first tile of each CTA's range in each level
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
// Counter updates that publish (release) everything this warp wrote before them (the
// __syncwarp() before each call orders the other lanes' writes first); the acquire-release
// form also makes every write published before the value it reads visible to the warp.
Q4_DEVINL void red_release_add(int *p, int v) {
    asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
Q4_DEVINL int atom_acq_rel_add(int *p, int v) {
    int old;
    asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
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

// The CTA that owns tile u of a level with U tiles.
Q4_DEVINL int cta_of(int64_t u, int64_t U, int G) { return (int)(((u + 1) * G - 1) / U); }

// Entry of tile u (level-local), searching forward from e.
Q4_DEVINL int locate(const StackEntry *ent, int e, int e_end, int64_t u) {
    while (e + 1 < e_end && u >= ent[e + 1].unit_base) ++e;
    return e;
}

// Position of a tile: GEMV e, row block rb, k-stage s.
struct Cursor {
    int e, rb, s;
};
Q4_DEVINL Cursor cursor_at(const StackEntry *ent, const StackLevel &lv, int64_t u) {
    Cursor cu;
    cu.e = locate(ent, lv.e0, lv.e0 + lv.ne, u);
    const int ul = (int)(u - ent[cu.e].unit_base);  // < R * S < 2^31
    const int S = ent[cu.e].S;
    cu.rb = ul / S;
    cu.s = ul - cu.rb * S;
    return cu;
}
// One tile forward; true when it moved to another GEMV (whose fields must be reloaded).
Q4_DEVINL bool cursor_next(Cursor &cu, int S, int R) {
    if (++cu.s < S) return false;
    cu.s = 0;
    if (++cu.rb < R) return false;
    cu.rb = 0;
    ++cu.e;
    return true;
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
__global__ void __maxnreg__(128) gemv_stack(const StackArgs a) {
    constexpr int SPS = kTileBytes / (4 * L);
    constexpr int KTI = BITS == 4 ? L / 2 : L / 4;
    constexpr int KTS = SPS * KTI;
    constexpr int WPT = L / 4;
    constexpr int STAGEK = kTileBytes * 8 / BITS;
    constexpr int GS = GPS > 0 ? GPS : 1;
    constexpr int FSLOT = slot1_bytes<BITS>();  // B fragments of one tile + format header
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint8_t *ring = smem;                                                  // kRing x 30 KB
    uint8_t *bbuf = ring + kRing * kSTile;                             // ucap x FSLOT
    uint64_t *full = reinterpret_cast<uint64_t *>(bbuf + (size_t)a.ucap * FSLOT);
    uint64_t *empty = full + kRing;
    int *flag = reinterpret_cast<int *>(empty + kRing);  // [0]: a wait of this CTA gave up

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int c = blockIdx.x, G = a.G;
    if (threadIdx.x == 0) {
        for (int i = 0; i < kRing; ++i) {
            mbar_init(full + i, 1);  // the TMA's expect_tx arrival
            mbar_init(empty + i, kConsumers);
        }
        flag[0] = 0;
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
            const int *us = a.ustart + (size_t)l * (G + 1);
            const int64_t u0 = us[c];
            const int n = us[c + 1] - us[c];
            if (n == 0) continue;
            Cursor cu = cursor_at(a.ent, lv, u0);
            const StackEntry *E = a.ent + cu.e;
            int S = E->S, R = E->R;
            tmap_acquire(&E->tm);
            for (int i = 0; i < n; ++i) {
                if (i > 0 && cursor_next(cu, S, R)) {
                    E = a.ent + cu.e;
                    S = E->S;
                    R = E->R;
                    tmap_acquire(&E->tm);
                }
                if (round > 0 && !timed_out) timed_out = !mbar_wait(empty + slot, (uint32_t)((round - 1) & 1), a.wait_ns);
                if (lane == 0 && !timed_out) {
                    mbar_arrive_expect_tx(full + slot, kSTile);
                    tma_load_2d_g(ring + slot * kSTile, &E->tm, full + slot, cu.s * kTileBytes, cu.rb * kSRows);
                }
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
        float ys0 = 0.f, ys1 = 0.f;  // this lane's share of rows pr and pr + 8
        int slot = 0, round = 0;
        for (int l = 0; l < a.L; ++l) {
            const StackLevel lv = a.lev[l];
            const int *us = a.ustart + (size_t)l * (G + 1);
            const int64_t u0 = us[c];
            const int n = us[c + 1] - us[c];
            if (n == 0) continue;
            if (l > 0) {
                // the activations of this level are complete once every warp of every row
                // block of the previous level has published its rows
                if (ct == 0 && !timed_out)
                    timed_out = !wait_counter(a.level_done + (l - 1), kConsumers * a.lev[l - 1].T, a.wait_ns);
                named_barrier_sync(1, kConsumerThreads);
            }
            // B fragments of tiles [i0, i1) of this level (i relative to u0), one tile per warp
            // at a time: exact integer digits or bf16 pieces, decided per tile
            auto build = [&](int i0, int i1) {
                for (int i = i0 + warp; i < i1; i += kConsumers) {
                    const Cursor bc = cursor_at(a.ent, lv, u0 + i);
                    const StackEntry *BE = a.ent + bc.e;
                    build_slot1<BITS, L, XBF16, true>(bbuf + (size_t)(i - i0) * FSLOT, BE->x, bc.s * STAGEK, BE->K,
                                                     a.P, lane);
                }
            };
            int chunk_lo = 0, chunk_hi = min(n, a.ucap);
            build(0, chunk_hi);
            named_barrier_sync(1, kConsumerThreads);

            Cursor cu = cursor_at(a.ent, lv, u0);
            const StackEntry *E = a.ent + cu.e;
            int S = E->S, R = E->R, N = E->N, K = E->K, task_base = E->task_base, spr = E->spr, group = E->group;
            float *y = E->y;
            const float *scales = E->scales;
            int64_t unit_base = E->unit_base;
            int seg_s0 = cu.s;  // first stage of the current row block in this CTA
            for (int i = 0; i < n; ++i) {
                if (i > 0) {
                    if (cursor_next(cu, S, R)) {
                        E = a.ent + cu.e;
                        S = E->S; R = E->R; N = E->N; K = E->K; task_base = E->task_base;
                        spr = E->spr; group = E->group;
                        y = E->y;
                        scales = E->scales;
                        unit_base = E->unit_base;
                    }
                    if (cu.s == 0) seg_s0 = 0;
                }
                if (i == chunk_hi) {
                    named_barrier_sync(1, kConsumerThreads);  // every warp is done with the last chunk
                    chunk_lo = i;
                    chunk_hi = min(n, i + a.ucap);
                    build(chunk_lo, chunk_hi);
                    named_barrier_sync(1, kConsumerThreads);
                }
                const int seg_hi = (K * BITS / 8) / (4 * L);  // segments per row
                const int nsl = min(SPS, seg_hi - cu.s * SPS);
                // this lane's scales of the tile (rows pr and pr + 8, the groups of the stage),
                // read through L1 (a 128-byte line of a row serves many consecutive stages);
                // their latency overlaps the wait for the tile
                float s0r[GS], s1r[GS];
                {
                    const int gbase = GPS > 0 ? cu.s * GPS : (cu.s * STAGEK) / group;
                    const int ng = min(GS, spr - gbase);
                    const float *sp0 = scales + (size_t)min(cu.rb * kSRows + pr, N - 1) * spr + gbase;
                    const float *sp1 = scales + (size_t)min(cu.rb * kSRows + pr + 8, N - 1) * spr + gbase;
#pragma unroll
                    for (int q = 0; q < GS; ++q) {
                        s0r[q] = q < ng ? __ldg(sp0 + q) : 0.f;
                        s1r[q] = q < ng ? __ldg(sp1 + q) : 0.f;
                    }
                }
                if (!timed_out) timed_out = !mbar_wait(full + slot, (uint32_t)(round & 1), a.wait_ns);
                const uint8_t *stg = ring + slot * kSTile;
                uint32_t A0[SPS][WPT], A1[SPS][WPT];
#pragma unroll
                for (int sl = 0; sl < SPS; ++sl) {
                    lds_words<L>(A0[sl], stg + aoff[sl]);
                    lds_words<L>(A1[sl], stg + aoff[sl] + 8 * kTileBytes);
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(empty + slot);  // the codes are in registers
                if (++slot == kRing) { slot = 0; ++round; }
                const uint8_t *slt = bbuf + (size_t)(i - chunk_lo) * FSLOT;
                const int *hdr = reinterpret_cast<const int *>(slt + slot1_data<BITS>());
                if (hdr[0]) {
                    const float fl = digit_lane_factor<BITS>(hdr[1], t);
                    if (nsl == SPS)
                        stage1_digits<BITS, L, GPS, true>(A0, A1, slt, lane, s0r, s1r, nsl, fl, ys0, ys1);
                    else
                        stage1_digits<BITS, L, GPS, false>(A0, A1, slt, lane, s0r, s1r, nsl, fl, ys0, ys1);
                } else {
                    if (nsl == SPS)
                        stage1_pieces<BITS, L, GPS, true>(A0, A1, slt, lane, s0r, s1r, nsl, ys0, ys1);
                    else
                        stage1_pieces<BITS, L, GPS, false>(A0, A1, slt, lane, s0r, s1r, nsl, ys0, ys1);
                }

                // ---- end of this CTA's share of row block rb: each warp finishes its 16 rows ----
                if (cu.s == S - 1 || i == n - 1) {
                    const int T = task_base + cu.rb;
                    const bool whole = cu.s == S - 1 && seg_s0 == 0;
                    // rows pr and pr + 8: the four lanes of each row add their shares
                    float r0 = ys0 + __shfl_xor_sync(0xffffffffu, ys0, 1);
                    float r1 = ys1 + __shfl_xor_sync(0xffffffffu, ys1, 1);
                    r0 += __shfl_xor_sync(0xffffffffu, r0, 2);
                    r1 += __shfl_xor_sync(0xffffffffu, r1, 2);
                    ys0 = ys1 = 0.f;
                    // lane 4g writes row pr (r0), lane 4g + 1 row pr + 8 (r1)
                    const int r = pr + 8 * (t & 1);
                    const float v = (t & 1) ? r1 : r0;
                    const bool writer = t < 2;
                    const int nrow = cu.rb * kSRows + r;
                    if (whole) {
                        if (writer && nrow < N) y[nrow] = v;
                        __syncwarp();
                        if (lane == 0) red_release_add(a.level_done + l, 1);
                    } else {
                        // the partial sums of a CTA's rows go to its slot 0 when the row block
                        // starts inside the CTA's range, else to slot 1 (a range holds parts of
                        // at most two split row blocks)
                        const int64_t tf = unit_base + (int64_t)cu.rb * S;
                        if (writer) a.partial[((size_t)c * 2 + (u0 >= tf ? 0 : 1)) * kSRows + r] = v;
                        __syncwarp();
                        // the CTAs holding parts of this row block (lanes take one each), and
                        // whether this warp is the last of them to arrive for its rows
                        const int cf = cta_of(tf, lv.U, G), clast = cta_of(tf + S - 1, lv.U, G);
                        int arrivals = 0;
                        for (int base = cf; base <= clast; base += 32) {
                            const int cc = base + lane;
                            const bool in = cc <= clast && us[cc] < us[cc + 1];
                            arrivals += __popc(__ballot_sync(0xffffffffu, in));
                        }
                        int last = 0;
                        if (lane == 0)
                            last = atom_acq_rel_add(a.task_cnt + (size_t)T * kConsumers + warp, 1) == arrivals - 1;
                        last = __shfl_sync(0xffffffffu, last, 0);
                        if (last) {
                            // lane j reads the 16 partial sums of CTA cf + j; the warp adds them
                            // in a fixed tree order (deterministic), 32 CTAs at a time in order;
                            // lane rr keeps row 16 * warp + rr
                            __syncwarp();
                            float mine = 0.f;
                            for (int base = cf; base <= clast; base += 32) {
                                const int cc = base + lane;
                                const bool in = cc <= clast && us[cc] < us[cc + 1];
                                float pv[16];
                                if (in) {
                                    const float4 *src = reinterpret_cast<const float4 *>(
                                        a.partial + ((size_t)cc * 2 + (us[cc] >= tf ? 0 : 1)) * kSRows + 16 * warp);
#pragma unroll
                                    for (int q = 0; q < 4; ++q) {
                                        const float4 f4 = __ldcg(src + q);
                                        pv[4 * q] = f4.x; pv[4 * q + 1] = f4.y; pv[4 * q + 2] = f4.z; pv[4 * q + 3] = f4.w;
                                    }
                                } else {
#pragma unroll
                                    for (int q = 0; q < 16; ++q) pv[q] = 0.f;
                                }
#pragma unroll
                                for (int rr = 0; rr < 16; ++rr) {
                                    float t2 = pv[rr];
#pragma unroll
                                    for (int m = 16; m >= 1; m >>= 1) t2 += __shfl_xor_sync(0xffffffffu, t2, m);
                                    if (lane == rr) mine = base == cf ? t2 : mine + t2;
                                }
                            }
                            const int nr = cu.rb * kSRows + 16 * warp + lane;
                            if (lane < 16 && nr < N) y[nr] = mine;
                            __syncwarp();
                            if (lane == 0) {
                                a.task_cnt[(size_t)T * kConsumers + warp] = 0;
                                red_release_add(a.level_done + l, 1);
                            }
                        }
                    }
                }
            }
        }
    }
    if (timed_out) flag[0] = 1;
    __syncthreads();
    if (threadIdx.x == 0) {
        if (flag[0]) {
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
                for (int i = 0; i < a.n_tasks * kConsumers; ++i) a.task_cnt[i] = 0;
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
    size_t off_ent, off_lev, off_cnt, off_done, off_misc, off_part, off_us, bytes;
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
        tasks += (g.N + kSRows - 1) / kSRows;
    }
    if (tasks > (int64_t)1 << 30) return Q4_ERR_UNSUPPORTED;
    lo->nlev = gv[count - 1].level + 1;
    lo->n_tasks = (int)tasks;
    lo->off_ent = 0;
    lo->off_lev = al256((size_t)count * sizeof(StackEntry));
    lo->off_cnt = lo->off_lev + al256((size_t)lo->nlev * sizeof(StackLevel));
    lo->off_done = lo->off_cnt + al256((size_t)lo->n_tasks * kConsumers * 4);
    lo->off_misc = lo->off_done + al256((size_t)lo->nlev * 4);
    lo->off_part = lo->off_misc + 256;
    lo->off_us = lo->off_part + al256((size_t)kPlanGrid * 2 * kSRows * 4);
    lo->bytes = lo->off_us + al256((size_t)lo->nlev * (kPlanGrid + 1) * 4);
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
            if (!encode_payload_map(&E.tm, g.payload, g.N, g.K, bits, kSRows)) return Q4_ERR_UNSUPPORTED;
            E.scales = g.scales;
            E.x = g.x;
            E.y = g.y;
            E.N = (int)g.N;
            E.K = (int)g.K;
            E.group = (int)g.group;
            E.spr = (int)(g.K / g.group);
            E.S = (int)((g.K * bits / 8 + kTileBytes - 1) / kTileBytes);
            E.R = (int)((g.N + kSRows - 1) / kSRows);
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
    const size_t fslot = bits == 4 ? slot1_bytes<4>() : slot1_bytes<8>();  // B fragments + header of a tile
    const int gsl = lo.gps > 0 ? lo.gps : 1;
    const size_t fixed = 1024 + (size_t)kRing * kSTile + 2 * kRing * 8 + 16;
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

    // each CTA's first tile in each level: an even split of the level's tiles
    std::vector<int> ustart((size_t)lo.nlev * (grid + 1));
    for (int l = 0; l < lo.nlev; ++l) {
        if (lev[l].U >= ((int64_t)1 << 31)) return Q4_ERR_UNSUPPORTED;
        for (int cc = 0; cc <= grid; ++cc) ustart[(size_t)l * (grid + 1) + cc] = (int)(lev[l].U * cc / grid);
    }
    // copy the tables, zero the counters; the host tables can go once the stream is done
    char *w = static_cast<char *>(workspace);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if ((e = cudaMemcpyAsync(w + lo.off_ent, ent.data(), ent.size() * sizeof(StackEntry), cudaMemcpyHostToDevice,
                             s)) != cudaSuccess ||
        (e = cudaMemcpyAsync(w + lo.off_lev, lev.data(), lev.size() * sizeof(StackLevel), cudaMemcpyHostToDevice,
                             s)) != cudaSuccess ||
        (e = cudaMemcpyAsync(w + lo.off_us, ustart.data(), ustart.size() * sizeof(int), cudaMemcpyHostToDevice,
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
    p.args.ustart = reinterpret_cast<const int *>(w + lo.off_us);
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
