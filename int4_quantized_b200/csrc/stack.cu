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
//   * The weight tiles (240 rows x 128 bytes) of a level are numbered GEMV by GEMV, row
//     block by row block, k-stage by k-stage, and each of the G resident CTAs takes one
//     contiguous G-th of them (an even split of the level's bytes, whatever its shapes).
//     Where a level has few row blocks, each row block is split over CTAs of its own
//     instead, when that keeps the longest range as short: then no range spans two row
//     blocks, and a row block has fewer parts.
//   * A producer warp per CTA streams the CTA's tiles of every level, in order, through
//     one TMA ring, and asks L2 for the scales each stretch of tiles will need. It never
//     waits for a level: the weights are static, so the next level's tiles arrive while
//     the current level ends.
//   * Fifteen consumer warps (16 rows of each tile apiece) wait (bounded, on a device
//     counter) until every part of the previous level is published, build the exact
//     digits or bf16 pieces of x for their tiles, and multiply. What a slot build needs
//     from the tables (which GEMV, where its x or parts are) is read before the wait, so
//     after it only the loads of x remain.
//   * A row block whose k-stages fall to several CTAs ends as several parts, one per
//     CTA, kept in a [parts][rows] matrix per GEMV; a part is published with one release
//     increment of the level's counter, without waiting for the other parts. Nobody
//     adds the parts up on the way to the next level: where a GEMV's x is a slice of a
//     previous-level GEMV's y, the next level reads x as the sum of that slice's parts
//     (in part order; absent parts are zeros). The y of a split row block is written by
//     the CTA holding its last part, as the same sum, so y and what the next level read
//     are the same numbers; it does so at the start of the level after next, on the warps
//     that have no slot to build while the others build (at the next start, before the
//     build, if the next level reads that y directly). Those warps post their release as a
//     ticket in shared memory; the producer warp takes it between two loads and makes the
//     GPU-scope release, so no consumer waits for the rows' stores to land. A level waits
//     for the sums of three levels back (the parts buffers rotate over three levels) and
//     of every earlier level whose y it reads directly.
//   * Counters return to zero at the end of every launch (the last CTA to finish resets
//     them), so the workspace can be replayed, e.g. from a CUDA graph.
//
// Every wait is bounded (about one second); one that gives up sets Q4_STATUS_TIMEOUT and
// the CTA goes on without waiting, so the launch always ends. Before a CTA exits, its
// producer waits (bounded) for every copy it issued into the CTA's shared memory.
#include <cuda.h>

#include <algorithm>
#include <cstring>
#include <vector>

#include "common.cuh"
#include "gemv_math.cuh"
#include "kernels.h"

namespace q4 {

namespace {

using namespace gm;

// One CTA per SM: fifteen consumer warps (16 weight rows each) on 240-row tiles and one
// producer warp. Registers: 512 threads x 128 fill the SM's 64K. The consumers read scales
// through L1 (a 128-byte line serves a row over many consecutive stages), so shared memory
// leaves room for it (below).
constexpr int kConsumers = 15;
constexpr int kConsumerThreads = 32 * kConsumers;
constexpr int kThreads = kConsumerThreads + 32;
constexpr int kSRows = 16 * kConsumers;            // 240 weight rows per tile
constexpr int kSTile = kTileBytes * kSRows;        // 30 KB of codes per tile
// Tiles in flight per CTA, and the shared memory the CTA takes: with several scale groups
// per tile the consumers' scale lines need about 70 KB of L1 (4 tiles, 160 KB of shared
// memory); with one scale per stage or per row they need little, and a fifth tile in
// flight pays (172 KB).
__host__ __device__ constexpr int ring_of(int gps) { return gps > 0 ? 4 : 5; }
constexpr int smem_budget_of(int gps) { return gps > 0 ? 163840 : 174080; }
constexpr int ucap_max_of(int gps) { return gps > 0 ? 64 : 10; }
constexpr int kCtasPerSm = 1;

struct alignas(64) StackEntry {
    CUtensorMap tm;        // 2D map of the payload: {row bytes, N}, box 128 x 240, 128B swizzle
    // consumer fields (one 128-byte line)
    const float *scales;
    const void *x;
    float *y;
    float *parts;          // [pmax][npad] the parts of this GEMV's row blocks
    const float *xparts;   // non-null: x is the sum over xpmax parts of these rows (stride xstride)
    int64_t unit_base;     // first tile of this GEMV in its level's numbering
    int N, K;
    int group;             // scale group (divides K)
    int spr;               // scales per row = K / group
    int S;                 // k-stages per row (128 bytes of payload each)
    int R;                 // row blocks of 240
    int pmax, npad;        // parts per row block at most; row stride of parts
    int xpmax, xstride;
    int is_src;            // the next level reads x from this GEMV's parts
    int level;
};

struct StackLevel {
    int64_t U;             // tiles in the level
    int e0, ne;            // its GEMVs
    int parts_target;      // parts that complete the level (one arrival per part)
    int fin_target;        // arrivals that complete its sums of split row blocks: one per block
    int fin_lo, fin_hi;    // levels whose sums must be in y before this level starts (none: lo > hi)
    int needs_final;       // the previous level's sums go to y at this level's start: it reads
                           // that y other than as a slice of parts, or the next level reads
                           // the y of the level before it
};

struct StackArgs {
    const StackEntry *ent;
    const StackLevel *lev;
    int *parts_done;       // [L] published (row block, part) pairs per level
    int *fin_done;         // [L] finished (split row block, warp) sums per level
    int *finished;         // CTAs done with the launch
    const int *ustart;     // [L][G + 1] first tile of each CTA's range in each level
    const int *pfirst;     // [L][G] part index of the row block each CTA's range starts in
    uint32_t *status;
    int G, L;
    int P;                 // pieces per activation: 3 (fp32 x) or 1 (bf16 x)
    int ucap;              // tiles whose activation pieces fit in shared memory at once
    uint64_t wait_ns;      // bound of every wait
};

Q4_DEVINL int ld_acquire(const int *p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
// A counter update that publishes (release) everything this warp wrote before it (the
// __syncwarp() before each call orders the other lanes' writes first).
Q4_DEVINL void red_release_add(int *p, int v) {
    asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
Q4_DEVINL int atom_exch_acq_rel_cta_shared(int *p, int v) {
    int old;
    asm volatile("atom.exch.acq_rel.cta.shared.b32 %0, [%1], %2;" : "=r"(old) : "r"(smem_u32(p)), "r"(v) : "memory");
    return old;
}
Q4_DEVINL int atom_acq_rel_cta_shared_add(int *p, int v) {
    int old;
    asm volatile("atom.acq_rel.cta.shared.add.s32 %0, [%1], %2;" : "=r"(old) : "r"(smem_u32(p)), "r"(v) : "memory");
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
Q4_DEVINL void prefetch_l2(const void *p) { asm volatile("prefetch.global.L2 [%0];" ::"l"(p)); }
Q4_DEVINL void prefetch_l1(const void *p) { asm volatile("prefetch.global.L1 [%0];" ::"l"(p)); }

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
        __nanosleep(32);
        if (ld_acquire(p) >= target) return true;
        if (global_ns() - t0 > limit_ns) return false;
    }
}

#ifndef Q4_STACK_MAX_READ_PARTS
#define Q4_STACK_MAX_READ_PARTS 1000
#endif
// A level reads x as the parts of the previous level's GEMV when each row has at most this
// many parts; with more, the reads cost more than waiting for the sums in y.
constexpr int kMaxReadParts = Q4_STACK_MAX_READ_PARTS;

// Warp-wide: every level j in [lo, hi] has all its sums of split row blocks in y (lane q
// watches level lo + q).
Q4_DEVINL bool wait_fin(const int *fin_done, const StackLevel *lev, int lo, int hi, uint64_t limit_ns, int lane) {
    for (int j0 = lo; j0 <= hi; j0 += 32) {
        const int j = j0 + lane;
        const int target = j <= hi ? lev[j].fin_target : 0;
        auto done = [&]() { return j > hi || ld_acquire(fin_done + j) >= target; };
        if (__all_sync(0xffffffffu, done())) continue;
        const uint64_t t0 = global_ns();
        for (;;) {
            __nanosleep(32);
            if (__all_sync(0xffffffffu, done())) break;
            if (__any_sync(0xffffffffu, global_ns() - t0 > limit_ns)) return false;
        }
    }
    return true;
}

// The output of a split row block's sum (see the consumers' finalize).
struct FinSrc {
    const float *parts;
    float *y;
    int N, npad, pmax, pad;
};

// Where the activations of a slot come from (see the consumers' slot build).
struct SlotSrc {
    const float *xp;  // non-null: x is the sum of these parts
    const void *x;    // otherwise x itself
    int k0, K;        // first k of the stage; K of the GEMV
    int pm, st4;      // parts; their row stride in float4
};

// First scale group of k-stage s.
template <int GPS, int STAGEK>
Q4_DEVINL int stage_group(int s, int group) {
    return GPS > 0 ? s * GPS : (s * STAGEK) / group;
}

template <int BITS, int L, int GPS, bool XBF16>
__global__ void __maxnreg__(128) gemv_stack(const StackArgs a) {
    constexpr int SPS = kTileBytes / (4 * L);
    constexpr int WPT = L / 4;
    constexpr int STAGEK = kTileBytes * 8 / BITS;
    constexpr int LANES = STAGEK / 8;
    // parts of x read at a time when a slot is built (measured: four for int4 codes; the
    // int8 kernel, tighter on registers, keeps two)
    constexpr int QB = BITS == 4 ? 4 : 2;
    constexpr int GS = GPS > 0 ? GPS : 1;
    constexpr int FSLOT = slot1_bytes<BITS>();  // B fragments of one tile + format header
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    constexpr int kRing = ring_of(GPS);
    uint8_t *ring = smem;                                                  // kRing x 30 KB
    uint8_t *bbuf = ring + kRing * kSTile;                             // ucap x FSLOT
    uint64_t *full = reinterpret_cast<uint64_t *>(bbuf + (size_t)a.ucap * FSLOT);
    uint64_t *empty = full + kRing;
    int *flag = reinterpret_cast<int *>(empty + kRing);  // [0]: a wait of this CTA gave up
    int *ticket = flag + 2;  // split-block sums written and not yet released: their level + 1
    // the GPU-scope release of a posted ticket (whoever takes it: the producer between its
    // loads, warp 0 before it waits, thread 0 at the end)
    auto take_ticket = [&]() {
        const int tk = atom_exch_acq_rel_cta_shared(ticket, 0);
        if (tk) red_release_add(a.fin_done + tk - 1, 1);
    };
    int *finq = flag + 4;  // [warp][2][4] pending sums of split row blocks: {entry, rb, parts, level}
    int *pubq = finq + kConsumers * 8;  // [8] warps arrived at each of the last eight publications
    SlotSrc *srcq = reinterpret_cast<SlotSrc *>(pubq + 8);  // [warp] its first slot's source
    FinSrc *fsrc = reinterpret_cast<FinSrc *>(srcq + kConsumers);  // level l - 2's block

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int c = blockIdx.x, G = a.G;
    if (threadIdx.x == 0) {
        for (int i = 0; i < kRing; ++i) {
            mbar_init(full + i, 1);  // the TMA's expect_tx arrival
            mbar_init(empty + i, kConsumers);
        }
        flag[0] = 0;
        flag[2] = 0;  // a posted release of split-block sums: its level + 1, or 0
        for (int i = 0; i < 8; ++i) pubq[i] = 0;
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
                if (lane == 0) take_ticket();
                if (round > 0 && !timed_out) timed_out = !mbar_wait(empty + slot, (uint32_t)((round - 1) & 1), a.wait_ns);
                if (lane == 0 && !timed_out) {
                    mbar_arrive_expect_tx(full + slot, kSTile);
                    tma_load_2d_g(ring + slot * kSTile, &E->tm, full + slot, cu.s * kTileBytes, cu.rb * kSRows);
                }
                ++issued[slot];
                if (++slot == kRing) { slot = 0; ++round; }
                if (i == 0 || cu.s == 0) {
                    // the scales of this CTA's stretch of the row block, into L2 ahead of use
                    const int s_end = min(S - 1, cu.s + (n - i) - 1);
                    const int g_lo = stage_group<GPS, STAGEK>(cu.s, E->group);
                    const int g_hi = min(E->spr - 1, stage_group<GPS, STAGEK>(s_end, E->group) + GS - 1);
                    const int N = E->N, spr = E->spr;
                    const float *sc = E->scales;
                    for (int rr = lane; rr < kSRows; rr += 32) {
                        const int row = cu.rb * kSRows + rr;
                        if (row >= N) break;
                        const uintptr_t lo = (uintptr_t)(sc + (size_t)row * spr + g_lo) & ~(uintptr_t)127;
                        const uintptr_t hi = (uintptr_t)(sc + (size_t)row * spr + g_hi);
                        for (uintptr_t q = lo; q <= hi; q += 128) prefetch_l2(reinterpret_cast<const void *>(q));
                    }
                }
            }
        }
        // drain: every copy issued into this CTA's shared memory has landed before it exits
#pragma unroll
        for (int i = 0; i < kRing; ++i)
            if (issued[i] > 0) (void)mbar_wait(full + i, (uint32_t)((issued[i] - 1) & 1), a.wait_ns);
    } else {
        // ---------------- consumers ----------------
        const int g = lane >> 2, t = lane & 3;

        const int pr = 16 * warp + row_perm<L>(g);
        uint32_t aoff[SPS];
#pragma unroll
        for (int sl = 0; sl < SPS; ++sl) {
            const int off = sl * 4 * L + t * L;
            aoff[sl] = pr * kTileBytes + (((off >> 4) ^ (pr & 7)) << 4) + (off & 15);
        }
        float ys0 = 0.f, ys1 = 0.f;  // this lane's share of rows pr and pr + 8
        int slot = 0, round = 0;
        int pub_j = 0;  // publications of this warp so far
        // split row blocks whose last part this CTA holds, by level parity: their sums (rows
        // of y) are written at the start of the level after next (see the file comment)
        int *fq = finq + warp * 8;
        if (lane == 0) fq[0] = fq[4] = -1;
        __syncwarp();
        // the sum of split row block f, parts in order, by warps w0..14 (the others are busy
        // building); one release for the block once all of them have written their rows
        auto fin_src = [&](const int *f) {
            const StackEntry *fe = a.ent + f[0];
            FinSrc r;
            r.parts = fe->parts;
            r.y = fe->y;
            r.N = fe->N;
            r.npad = fe->npad;
            r.pmax = fe->pmax;
            r.pad = 0;
            return r;
        };
        auto finalize = [&](const int *f, const FinSrc fe, int w0, bool post) {
            if (warp < w0) return;
            const int nw = kConsumers - w0;
            const int np = f[2];
            const size_t st = (size_t)fe.npad;
            for (int rr = (warp - w0) * 32 + lane; rr < kSRows; rr += nw * 32) {
                const int row = f[1] * kSRows + rr;
                if (row < fe.N) {
                    // twelve loads in flight at a time, added in part order
                    const float *pp = fe.parts + row;
                    float v = 0.f;
                    for (int q0 = 0; q0 < np; q0 += 12) {
                        float pv[12];
#pragma unroll
                        for (int j = 0; j < 12; ++j) pv[j] = q0 + j < np ? __ldcg(pp + (q0 + j) * st) : 0.f;
#pragma unroll
                        for (int j = 0; j < 12; ++j)
                            if (q0 + j < np) v = q0 + j == 0 ? pv[0] : v + pv[j];
                    }
                    if (np < fe.pmax) v += 0.f;  // as the sum over all pmax parts, zeros included
                    fe.y[row] = v;
                }
            }
            named_barrier_sync(2, nw * 32);
            if (warp == w0 && lane == 0) {
                if (post) {
                    // a CTA-scope release of the rows to whoever takes the ticket, so these
                    // warps do not wait for their stores to land (an older ticket still
                    // posted is released here)
                    const int old = atom_exch_acq_rel_cta_shared(ticket, f[3] + 1);
                    if (old) red_release_add(a.fin_done + old - 1, 1);
                } else {
                    __threadfence();
                    red_release_add(a.fin_done + f[3], 1);
                }
            }
        };
        for (int l = 0; l <= a.L; ++l) {
            int64_t u0 = 0;
            int n = 0, pcur = 0;
            if (l < a.L) {
                const int *us = a.ustart + (size_t)l * (G + 1);
                u0 = us[c];
                n = us[c + 1] - us[c];
                pcur = a.pfirst[(size_t)l * G + c];
            }
            int *f_old = fq + 4 * (l & 1);        // a block of level l - 2
            int *f_new = fq + 4 * ((l + 1) & 1);  // a block of level l - 1
            const bool has_old = f_old[0] >= 0, has_new = f_new[0] >= 0;
            if (n == 0 && !has_old && !has_new) continue;
            StackLevel lv;
            Cursor cu;
            if (l < a.L) lv = a.lev[l];
            // where the x of tile i (relative to u0) comes from: the tables only, so a warp
            // reads its first slot's before the wait for the previous level
            auto slot_src = [&](int i) {
                SlotSrc r;
                const Cursor bc = cursor_at(a.ent, lv, u0 + i);
                const StackEntry *BE = a.ent + bc.e;
                r.xp = XBF16 ? nullptr : BE->xparts;
                r.x = BE->x;
                r.k0 = bc.s * STAGEK;
                r.K = BE->K;
                r.pm = BE->xpmax;
                r.st4 = BE->xstride / 4;
                return r;
            };
            // the entry of level l - 2's block, read while the level waits
            if (has_old && warp == kConsumers - 1 && lane == 0) *fsrc = fin_src(f_old);
            const bool has_first = n > 0 && warp < min(n, a.ucap);
            if (has_first) {
                const SlotSrc f = slot_src(warp);
                if (lane == 0) srcq[warp] = f;
            }
            if (n > 0) {
                cu = cursor_at(a.ent, lv, u0);
                // the first tile's scale lines, into L1 while this level waits
                const StackEntry *E0 = a.ent + cu.e;
                const int gb = stage_group<GPS, STAGEK>(cu.s, E0->group);
                const int N0 = E0->N;
                prefetch_l1(E0->scales + (size_t)min(cu.rb * kSRows + pr, N0 - 1) * E0->spr + gb);
                prefetch_l1(E0->scales + (size_t)min(cu.rb * kSRows + pr + 8, N0 - 1) * E0->spr + gb);
            }
            if (l > 0) {
                // the activations are complete once every warp of every part of the previous
                // level has published its rows, and the levels this one needs have their sums
                if (warp == 0 && !timed_out) {
                    bool ok = true;
                    if (lane == 0) take_ticket();  // never wait on sums of this CTA's own not yet released
                    __syncwarp();
                    // the sums first: they are older and usually long in y, so their check
                    // is over before the previous level ends
                    if (l < a.L) ok = wait_fin(a.fin_done, a.lev, lv.fin_lo, lv.fin_hi, a.wait_ns, lane);
                    if (ok && lane == 0) ok = wait_counter(a.parts_done + (l - 1), a.lev[l - 1].parts_target, a.wait_ns);
                    ok = __shfl_sync(0xffffffffu, ok, 0);
                    timed_out = !ok;
                }
                named_barrier_sync(1, kConsumerThreads);
            }
            // pending sums: level l - 2's blocks (their parts were complete before level l - 1
            // started) and level l - 1's (complete now), the latter only when this level reads
            // their y, or has no tiles, or is the end. Warps with no slot to build do them
            // while the others build.
            const bool now_new = has_new && (l == a.L || n == 0 || lv.needs_final);
            const int w_free = (l == a.L || n == 0 || lv.needs_final) ? 0 : min(kConsumers, min(n, a.ucap));
            if (w_free < kConsumers) {
                if (has_old) finalize(f_old, *fsrc, w_free, l < a.L && n > 0);
                if (now_new) finalize(f_new, fin_src(f_new), w_free, false);
            }
            if (lane == 0) {
                if (has_old && w_free < kConsumers) f_old[0] = -1;
                if (now_new) f_new[0] = -1;
            }
            __syncwarp();
            if (l == a.L || n == 0) continue;
            if (lv.needs_final) {
                named_barrier_sync(1, kConsumerThreads);
                if (warp == 0 && !timed_out) timed_out = !wait_fin(a.fin_done, a.lev, l - 1, l - 1, a.wait_ns, lane);
                named_barrier_sync(1, kConsumerThreads);
            }
            // B fragments of tiles [i0, i1) of this level (i relative to u0), one tile per warp
            // at a time: exact integer digits or bf16 pieces, decided per tile
            auto build = [&](int i0, int i1) {
                for (int i = i0 + warp; i < i1; i += kConsumers) {
                    const SlotSrc src = i0 == 0 && i == warp ? srcq[warp] : slot_src(i);
                    uint8_t *bs = bbuf + (size_t)(i - i0) * FSLOT;
                    const float *xp = src.xp;
                    if (!xp) {
                        build_slot1<BITS, L, XBF16, true>(bs, src.x, src.k0, src.K, a.P, lane);
                        continue;
                    }
                    // x = the sum of the producing GEMV's parts of these rows, in part order
                    float v[8];
#pragma unroll
                    for (int q = 0; q < 8; ++q) v[q] = 0.f;
                    const int k = src.k0 + 8 * lane;
                    if (lane < LANES && k < src.K) {
                        const float4 *xq = reinterpret_cast<const float4 *>(xp + k);
                        const size_t st4 = (size_t)src.st4;
                        const int pm = src.pm;
                        float4 s0 = __ldcg(xq), s1 = __ldcg(xq + 1);
                        // QB parts in flight at a time, added in part order
                        for (int q0 = 1; q0 < pm; q0 += QB) {
                            float4 b[QB][2];
#pragma unroll
                            for (int j = 0; j < QB; ++j) {
                                b[j][0] = b[j][1] = make_float4(0.f, 0.f, 0.f, 0.f);
                                if (q0 + j < pm) {
                                    b[j][0] = __ldcg(xq + (q0 + j) * st4);
                                    b[j][1] = __ldcg(xq + (q0 + j) * st4 + 1);
                                }
                            }
#pragma unroll
                            for (int j = 0; j < QB; ++j)
                                if (q0 + j < pm) {
                                    s0.x += b[j][0].x; s0.y += b[j][0].y; s0.z += b[j][0].z; s0.w += b[j][0].w;
                                    s1.x += b[j][1].x; s1.y += b[j][1].y; s1.z += b[j][1].z; s1.w += b[j][1].w;
                                }
                        }
                        v[0] = s0.x; v[1] = s0.y; v[2] = s0.z; v[3] = s0.w;
                        v[4] = s1.x; v[5] = s1.y; v[6] = s1.z; v[7] = s1.w;
                    }
                    build_slot1_v<BITS, L>(bs, v, a.P, lane);
                }
            };
            int chunk_lo = 0, chunk_hi = min(n, a.ucap);
            build(0, chunk_hi);
            if (has_old && w_free == kConsumers) {  // every warp built: the sum comes after
                finalize(f_old, *fsrc, 0, true);
                if (lane == 0) f_old[0] = -1;
                __syncwarp();
            }
            named_barrier_sync(1, kConsumerThreads);

            const StackEntry *E = a.ent + cu.e;
            int S = E->S, R = E->R, N = E->N, K = E->K, spr = E->spr, group = E->group;
            const float *scales = E->scales;
            int pend = 0;  // parts written and not yet published
            for (int i = 0; i < n; ++i) {
                if (i > 0) {
                    if (cursor_next(cu, S, R)) {
                        E = a.ent + cu.e;
                        S = E->S; R = E->R; N = E->N; K = E->K;
                        spr = E->spr; group = E->group;
                        scales = E->scales;
                    }
                    if (cu.s == 0) pcur = 0;  // a row block that starts in this CTA's range
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
                    const int gbase = stage_group<GPS, STAGEK>(cu.s, group);
                    const int ng = min(GS, spr - gbase);
                    const float *sp0 = scales + (size_t)min(cu.rb * kSRows + pr, N - 1) * spr + gbase;
                    const float *sp1 = scales + (size_t)min(cu.rb * kSRows + pr + 8, N - 1) * spr + gbase;
                    // four groups a stage (g64 int4): one vector load per row when they are
                    // whole and aligned (measured: with two groups the vector form makes the
                    // kernel spill)
                    const bool vec = GS == 4 && ng == GS &&
                                     ((reinterpret_cast<uintptr_t>(sp0) | reinterpret_cast<uintptr_t>(sp1)) & 15u) == 0;
                    if (vec) {
                        if constexpr (GS == 4) {
                            const float4 v0 = __ldg(reinterpret_cast<const float4 *>(sp0));
                            const float4 v1 = __ldg(reinterpret_cast<const float4 *>(sp1));
                            s0r[0] = v0.x; s0r[1] = v0.y; s0r[2] = v0.z; s0r[3] = v0.w;
                            s1r[0] = v1.x; s1r[1] = v1.y; s1r[2] = v1.z; s1r[3] = v1.w;
                        }
                    } else {
#pragma unroll
                        for (int q = 0; q < GS; ++q) {
                            s0r[q] = q < ng ? __ldg(sp0 + q) : 0.f;
                            s1r[q] = q < ng ? __ldg(sp1 + q) : 0.f;
                        }
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

                // ---- end of this CTA's part of row block rb: each warp publishes its 16 rows ----
                const bool block_end = cu.s == S - 1 || i == n - 1;
                if (block_end) {
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
                    const bool last_part = cu.s == S - 1;  // the row block ends in this CTA's range
                    const bool src = E->is_src != 0;
                    if (writer && nrow < N) {
                        if (last_part && pcur == 0) E->y[nrow] = v;  // the whole row block: v is y
                        if (pcur > 0 || !last_part || src) {
                            float *pp = E->parts + nrow;
                            const size_t st = (size_t)E->npad;
                            pp[pcur * st] = v;
                            if (last_part && src)
                                for (int q = pcur + 1; q < E->pmax; ++q) pp[q * st] = 0.f;
                        }
                    }
                    ++pend;
                    if (last_part && pcur > 0 && lane == 0) {
                        int *f = fq + 4 * (l & 1);  // summed at the start of level l + 2
                        f[0] = cu.e;
                        f[1] = cu.rb;
                        f[2] = pcur + 1;
                        f[3] = l;
                    }
                }
                // parts are published one tile late (their stores have landed by then, so the
                // release does not stall), and at once at the end of the CTA's range
                if (pend > 0 && (!block_end || i == n - 1)) {
                    // every warp publishes the same parts in the same order: the warps count
                    // their arrivals in shared memory and the last of the fifteen makes one
                    // release increment for the CTA (its release carries what the other warps
                    // wrote before their arrivals, which it acquired)
                    __syncwarp();
                    if (lane == 0) {
                        int *ctr = pubq + (pub_j & 7);
                        if (atom_acq_rel_cta_shared_add(ctr, 1) == kConsumers - 1) {
                            *ctr = 0;  // reused eight publications later; no warp is that far ahead
                            red_release_add(a.parts_done + l, pend);
                        }
                    }
                    ++pub_j;
                    pend = 0;
                }
            }
        }
    }
    if (timed_out) flag[0] = 1;
    __syncthreads();
    if (threadIdx.x == 0) {
        take_ticket();
        if (flag[0] && a.status) atomicOr(a.status, Q4_STATUS_TIMEOUT);
        __threadfence();
        const int old = atomicAdd(a.finished, 1);
        if (old == G - 1) {
            // every CTA is done with the counters: return them to zero for the next launch
            __threadfence();
            for (int l = 0; l < a.L; ++l) {
                a.parts_done[l] = 0;
                a.fin_done[l] = 0;
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

constexpr int kPlanGrid = 148 * kCtasPerSm;  // the workspace is sized for a full B200
constexpr uint64_t kPlanMagic = 0x71347374616b3032ull;

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

inline int64_t stages_of(int64_t K, int bits) { return (K * bits / 8 + kTileBytes - 1) / kTileBytes; }
inline int64_t blocks_of(int64_t N) { return (N + kSRows - 1) / kSRows; }
inline int64_t npad_of(int64_t N) { return (N + 3) / 4 * 4; }

// At most how many CTA ranges a row block of S tiles meets when a level of U tiles is
// split over G CTAs: ranges are at least max(1, U / G) tiles long. The bound only falls
// as G falls, so the workspace sized with the largest grid serves every smaller one.
inline int64_t parts_bound(int64_t S, int64_t U, int64_t G) {
    const int64_t m = std::max<int64_t>(1, U / G);
    return std::min<int64_t>(S, 1 + (S - 1 + m - 1) / m);
}

struct StackLayout {
    int L, gps, nlev;
    size_t part_floats;  // floats of one parts buffer (three rotate over the levels)
    size_t off_ent, off_lev, off_cnt, off_part, off_us, off_pf, bytes;
};

q4_status stack_layout(const q4_stack_gemv *gv, int32_t count, int bits, q4_xdtype xt, StackLayout *lo) {
    if (!gv || count < 1 || (bits != 4 && bits != 8) || (xt != Q4_X_F32 && xt != Q4_X_BF16)) return Q4_ERR_ARG;
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
    }
    lo->nlev = gv[count - 1].level + 1;
    // the largest parts buffer any level needs on any grid up to a full B200
    size_t pmax_floats = 0;
    for (int32_t i = 0; i < count;) {
        int32_t j = i;
        int64_t U = 0;
        for (; j < count && gv[j].level == gv[i].level; ++j) U += blocks_of(gv[j].N) * stages_of(gv[j].K, bits);
        if (U >= ((int64_t)1 << 31)) return Q4_ERR_UNSUPPORTED;
        size_t f = 0;
        for (int32_t e = i; e < j; ++e)
            f += (size_t)parts_bound(stages_of(gv[e].K, bits), U, kPlanGrid) * (size_t)npad_of(gv[e].N);
        pmax_floats = std::max(pmax_floats, f);
        i = j;
    }
    lo->part_floats = pmax_floats;
    lo->off_ent = 0;
    lo->off_lev = al256((size_t)count * sizeof(StackEntry));
    lo->off_cnt = lo->off_lev + al256((size_t)lo->nlev * sizeof(StackLevel));       // parts_done, fin_done, finished
    lo->off_part = lo->off_cnt + al256((size_t)(2 * lo->nlev + 1) * 4);
    lo->off_us = lo->off_part + 3 * al256(pmax_floats * 4);
    lo->off_pf = lo->off_us + al256((size_t)lo->nlev * (kPlanGrid + 1) * 4);
    lo->bytes = lo->off_pf + al256((size_t)lo->nlev * kPlanGrid * 4);
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

    // grid and shared memory
    const size_t fslot = bits == 4 ? slot1_bytes<4>() : slot1_bytes<8>();  // B fragments + header of a tile
    const int kRing = ring_of(lo.gps);
    const size_t budget = (size_t)smem_budget_of(lo.gps);
    const size_t fixed = 1024 + (size_t)kRing * kSTile + 2 * kRing * 8 + 16 + kConsumers * 8 * 4 + 8 * 4 +
                         kConsumers * sizeof(SlotSrc) + sizeof(FinSrc);
    if (fixed + fslot > budget) return Q4_ERR_UNSUPPORTED;
    int ucap = (int)((budget - fixed) / fslot);
    if (ucap > ucap_max_of(lo.gps)) ucap = ucap_max_of(lo.gps);
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

    char *w = static_cast<char *>(workspace);
    float *parts_buf[3];
    for (int q = 0; q < 3; ++q) parts_buf[q] = reinterpret_cast<float *>(w + lo.off_part + q * al256(lo.part_floats * 4));
    std::vector<StackEntry> ent(count);
    std::vector<StackLevel> lev(lo.nlev);
    std::vector<int> ustart((size_t)lo.nlev * (grid + 1));
    std::vector<int> pfirst((size_t)lo.nlev * grid, 0);
    for (int l = 0, i = 0; l < lo.nlev; ++l) {
        StackLevel &lv = lev[l];
        std::memset(&lv, 0, sizeof lv);
        lv.e0 = i;
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
            E.S = (int)stages_of(g.K, bits);
            E.R = (int)blocks_of(g.N);
            E.npad = (int)npad_of(g.N);
            E.level = l;
            E.unit_base = lv.U;
            lv.U += (int64_t)E.R * E.S;
        }
        lv.ne = i - lv.e0;
        // each CTA's first tile: an even split of the level's tiles, every range non-empty
        // when there are at least as many tiles as CTAs (else one tile for each of the first U)
        int *us = ustart.data() + (size_t)l * (grid + 1);
        for (int cc = 0; cc <= grid; ++cc)
            us[cc] = lv.U < grid ? (int)std::min<int64_t>(cc, lv.U) : (int)(lv.U * cc / grid);
        // where row blocks are few: each row block split over its own CTAs instead, when that
        // keeps the longest range as short (no range spans two row blocks, so a row block
        // has fewer parts for the next level to read)
        if (lv.U >= grid) {
            const int64_t longest = (lv.U + grid - 1) / grid;
            int64_t need = 0;
            for (int ei = lv.e0; ei < lv.e0 + lv.ne; ++ei)
                need += (int64_t)ent[ei].R * ((ent[ei].S + longest - 1) / longest);
            if (need <= grid) {
                int cc = 0;
                for (int ei = lv.e0; ei < lv.e0 + lv.ne; ++ei) {
                    const StackEntry &E = ent[ei];
                    const int c_rb = (int)((E.S + longest - 1) / longest);  // CTAs per row block
                    for (int rb = 0; rb < E.R; ++rb)
                        for (int q = 0; q < c_rb; ++q)
                            us[cc++] = (int)(E.unit_base + (int64_t)rb * E.S + (int64_t)E.S * q / c_rb);
                }
                for (; cc <= grid; ++cc) us[cc] = (int)lv.U;  // the CTAs left over have no tiles
            }
        }
        auto cta_of = [&](int64_t u) {  // the CTA whose range holds tile u
            return (int)(std::upper_bound(us, us + grid + 1, (int)u) - us) - 1;
        };
        // parts of every row block; this level's parts buffer (by level parity)
        size_t off = 0;
        int64_t pairs = 0, split = 0;
        for (int ei = lv.e0; ei < lv.e0 + lv.ne; ++ei) {
            StackEntry &E = ent[ei];
            int pm = 1;
            for (int rb = 0; rb < E.R; ++rb) {
                const int64_t tf = E.unit_base + (int64_t)rb * E.S;
                const int np = cta_of(tf + E.S - 1) - cta_of(tf) + 1;
                pm = std::max(pm, np);
                pairs += np;
                split += np > 1;
            }
            E.pmax = pm;
            E.parts = parts_buf[l % 3] + off;
            off += (size_t)pm * E.npad;
        }
        if (off > lo.part_floats) return Q4_ERR_WORKSPACE;  // cannot happen with grid <= kPlanGrid
        if (pairs >= ((int64_t)1 << 31)) return Q4_ERR_UNSUPPORTED;
        lv.parts_target = (int)pairs;
        lv.fin_target = (int)split;
        for (int cc = 0; cc < grid; ++cc) {
            if (us[cc] == us[cc + 1]) continue;
            int ei = lv.e0;
            while (ei + 1 < lv.e0 + lv.ne && us[cc] >= ent[ei + 1].unit_base) ++ei;
            const int64_t tf = ent[ei].unit_base + (us[cc] - ent[ei].unit_base) / ent[ei].S * ent[ei].S;
            pfirst[(size_t)l * grid + cc] = cc - cta_of(tf);
        }
    }
    // x of level l read as the parts of a level l - 1 GEMV whose y holds it (fp32, 16-byte
    // aligned slice). x overlapping the y of level l - 1 any other way: that level writes
    // its sums at the next start and level l waits for them; overlapping the y of an older
    // level: level l waits for that level's sums. Every level waits for the sums of three
    // levels back (the parts buffers rotate over three levels).
    for (int l = 0; l < lo.nlev; ++l) {
        lev[l].fin_lo = l >= 3 ? l - 3 : 0;
        lev[l].fin_hi = l >= 3 ? l - 3 : -1;
    }
    for (int i = 0; i < count; ++i) {
        StackEntry &E = ent[i];
        const int l = E.level;
        const uintptr_t x0 = (uintptr_t)E.x;
        const uintptr_t x1 = x0 + (uintptr_t)E.K * (bf16 ? 2 : 4);
        for (int j = 0; j < lev[l].e0; ++j) {
            StackEntry &P = ent[j];
            const uintptr_t y0 = (uintptr_t)P.y, y1 = y0 + (uintptr_t)P.N * 4;
            if (x1 <= y0 || x0 >= y1) continue;
            if (P.level == l - 1) {
                if (!bf16 && !E.xparts && x0 >= y0 && x1 <= y1 && (x0 - y0) % 16 == 0 && P.pmax <= kMaxReadParts) {
                    E.xparts = P.parts + (x0 - y0) / 4;
                    E.xpmax = P.pmax;
                    E.xstride = P.npad;
                    P.is_src = 1;
                } else {
                    lev[l].needs_final = 1;
                }
            } else {
                StackLevel &lv = lev[l];
                if (lv.fin_hi < lv.fin_lo) {
                    lv.fin_lo = lv.fin_hi = P.level;
                } else {
                    lv.fin_lo = std::min(lv.fin_lo, P.level);
                    lv.fin_hi = std::max(lv.fin_hi, P.level);
                }
                // the sums of level l - 2 are otherwise written at the start of level l,
                // after its wait for them: level l - 1 writes them at its start instead
                if (P.level == l - 2) lev[l - 1].needs_final = 1;
            }
        }
    }
    // copy the tables, zero the counters; the host tables can go once the stream is done
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if ((e = cudaMemcpyAsync(w + lo.off_ent, ent.data(), ent.size() * sizeof(StackEntry), cudaMemcpyHostToDevice,
                             s)) != cudaSuccess ||
        (e = cudaMemcpyAsync(w + lo.off_lev, lev.data(), lev.size() * sizeof(StackLevel), cudaMemcpyHostToDevice,
                             s)) != cudaSuccess ||
        (e = cudaMemcpyAsync(w + lo.off_us, ustart.data(), ustart.size() * sizeof(int), cudaMemcpyHostToDevice,
                             s)) != cudaSuccess ||
        (e = cudaMemcpyAsync(w + lo.off_pf, pfirst.data(), pfirst.size() * sizeof(int), cudaMemcpyHostToDevice,
                             s)) != cudaSuccess ||
        (e = cudaMemsetAsync(w + lo.off_cnt, 0, lo.off_part - lo.off_cnt, s)) != cudaSuccess ||
        (e = cudaStreamSynchronize(s)) != cudaSuccess)
        return cuda_error(e, "stack tables");

    StackPlanImpl p = {};
    p.magic = kPlanMagic;
    p.kern = kern;
    p.args.ent = reinterpret_cast<const StackEntry *>(w + lo.off_ent);
    p.args.lev = reinterpret_cast<const StackLevel *>(w + lo.off_lev);
    p.args.parts_done = reinterpret_cast<int *>(w + lo.off_cnt);
    p.args.fin_done = p.args.parts_done + lo.nlev;
    p.args.finished = p.args.fin_done + lo.nlev;
    p.args.ustart = reinterpret_cast<const int *>(w + lo.off_us);
    p.args.pfirst = reinterpret_cast<const int *>(w + lo.off_pf);
    p.args.status = nullptr;
    p.args.G = grid;
    p.args.L = lo.nlev;
    p.args.P = bf16 ? 1 : 3;
    p.args.ucap = ucap;
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
