// qpack.cu -- quantize+pack (K1) and dequantize (K2) kernels.
//
// The rule is pack()/unpack() of the page "量化推理：INT8/INT4 的体积、困惑度与速度
// 为什么不同步" (and "Huit bits, puis quatre", section "Arrondir"): per group of g
// consecutive weights of the flattened tensor, scale = fp32(absmax / qmax), 0 -> 1,
// code = clip(rint(w / scale), -qmax, qmax); int4 bytes hold (code+8) pairs with the
// even element in the low nibble. Each code equals rint of the IEEE round-to-nearest
// fp32 quotient (see code_fast for how most weights avoid a full division while
// staying bit-identical), so the output is bit-identical to the definition.
//
// Kernels:
//   qpack_chunk<BITS, G>    groups of 16..1024 that divide 1024: a warp quantizes 1024
//                           weights per step with coalesced 128-bit loads, shuffle
//                           reductions of the magnitude bits and 128-bit stores of the
//                           packed bytes (through a small shared-memory transpose).
//   qpack_group_cta<BITS,NQ> one CTA of 256 threads per group (large g, e.g. one scale
//                           per output channel): coalesced loads, the group stays in
//                           registers, the absmax is a block reduction.
//   qpack_generic_*         any group size / alignment: scales (one warp per group),
//                           then codes (one thread per output byte).
//   qdequant_vec / _generic w' = float(code) * scale.
#include "common.cuh"
#include "kernels.h"

namespace q4 {

namespace {

constexpr uint32_t kAbsMask = 0x7fffffffu;
constexpr uint32_t kInfBits = 0x7f800000u;

// |w| as bits: for non-negative floats (and NaN payloads above Inf) the unsigned
// integer order is the numeric order, so an integer max gives max|w| and
// flags any Inf/NaN (bits >= 0x7f800000) at the same time.
Q4_DEVINL uint32_t absbits(float v) { return __float_as_uint(v) & kAbsMask; }

template <int BITS>
Q4_DEVINL float scale_of(uint32_t maxbits) {
    constexpr float qmax = (float)((1 << (BITS - 1)) - 1);
    float s = __fdiv_rn(__uint_as_float(maxbits), qmax);
    return s == 0.0f ? 1.0f : s;
}

template <int BITS>
Q4_DEVINL int code_of(float w, float s) {
    constexpr float qmax = (float)((1 << (BITS - 1)) - 1);
    float r = rintf(__fdiv_rn(w, s));
    r = fminf(fmaxf(r, -qmax), qmax);
    return (int)r;
}

// code = clip(rint(RN(w / s))) without a full division per weight.
// Per group: r = RN(1/s). Per weight: q0 = RN(w r); e = RN(w - q0 s) (one fma);
// q1 = RN(q0 + e r) (one fma). One Newton-style correction of the reciprocal product
// leaves |q1 - w/s| within half an ulp plus a term below 2^-44 |w/s| (the classic
// reciprocal-and-residual division, P. Markstein, "IA-64 and Elementary Functions",
// 2000), so |q1 - RN(w/s)| is at most one ulp of the quotient: 2^-17 when
// |w/s| < 128 (int8), 2^-20 when |w/s| < 8 (int4); a subnormal residual adds at most
// 2^-25 for scales >= 2^-125. If q1 lies farther than kTie from every half-integer,
// RN(w/s) is inside the same rounding interval, so rint gives the same code; kTie is
// 16x those bounds. Otherwise (about 0.02 % of int8 and 0.003 % of int4 weights), and
// for scales outside [2^-125, 2^125) or non-finite values, the four weights of that
// float4 are recomputed with the correctly rounded IEEE division. The result is
// bit-identical to the definition.
// Rounding uses the magic constant 1.5 * 2^23 (+8 for int4): RN(q1 + C) = C + rint(q1)
// for |q1| < 2^22, so the code (int8) or the nibble code + 8 (int4) is in the low bits
// of the sum and no float-to-int conversion is needed. For finite inputs
// |w/s| <= qmax (1 + 2^-22), so rint never leaves [-qmax, qmax] and the clip is a no-op
// on this path; the exact path clips explicitly.
struct GroupDiv {
    float s, r;
    bool fast;
};
Q4_DEVINL GroupDiv make_div(float s) {
    GroupDiv d;
    d.s = s;
    d.fast = s >= 0x1p-125f && s < 0x1p125f;
    d.r = d.fast ? __frcp_rn(s) : 0.f;
    return d;
}
template <int BITS>
struct Magic {
    static constexpr float C = BITS == 4 ? 12582920.0f : 12582912.0f;  // 1.5*2^23 (+8)
    static constexpr float kTie = BITS == 4 ? 0x1p-16f : 0x1p-13f;
};
// Bits whose low nibble (int4: code + 8) or low byte (int8: code) are the packed value.
template <int BITS>
Q4_DEVINL uint32_t code_exact_bits(float w, float s, bool &nonfinite) {
    constexpr float qmax = (float)((1 << (BITS - 1)) - 1);
    nonfinite |= !isfinite(w) || !isfinite(s);
    float c = rintf(__fdiv_rn(w, s));
    c = fminf(fmaxf(c, -qmax), qmax);
    return __float_as_uint(c + Magic<BITS>::C);
}
// Four weights at once; the exact fallback runs for the whole float4 if any needs it.
template <int BITS>
Q4_DEVINL void codes4(const float (&w)[4], const GroupDiv &d, uint32_t (&t)[4], bool &nonfinite) {
    constexpr float C = Magic<BITS>::C;
    bool bad = !d.fast;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float q0 = w[i] * d.r;
        const float e = fmaf(-q0, d.s, w[i]);
        const float q1 = fmaf(e, d.r, q0);
        const float tt = q1 + C;
        const float cf = tt - C;
        bad |= !(fabsf(q1 - cf) <= 0.5f - Magic<BITS>::kTie);  // also true for NaN
        t[i] = __float_as_uint(tt);
    }
    if (bad) {
#pragma unroll
        for (int i = 0; i < 4; ++i) t[i] = code_exact_bits<BITS>(w[i], d.s, nonfinite);
    }
}
// Four codes -> 16 bits (int4: four nibbles, element 0 lowest) or 32 bits (int8).
template <int BITS>
Q4_DEVINL uint32_t pack4(const uint32_t (&t)[4]) {
    if constexpr (BITS == 4) {
        const uint32_t b = prmt(prmt(t[0], t[1], 0x0040u), prmt(t[2], t[3], 0x0040u), 0x5410u);
        // b = bytes (t0, t1, t2, t3); keep low nibbles: n0 | n1 << 4 | n2 << 8 | n3 << 12
        const uint32_t n = b & 0x0f0f0f0fu;
        const uint32_t m = (n | (n >> 4)) & 0x00ff00ffu;  // (n0|n1<<4, n2|n3<<4) in bytes 0, 2
        return prmt(m, 0u, 0x4420u);                     // bytes 0, 2 -> 16 bits
    } else {
        return prmt(prmt(t[0], t[1], 0x0040u), prmt(t[2], t[3], 0x0040u), 0x5410u);
    }
}
Q4_DEVINL float absmax4(float a, float b, float c, float d) {
    return fmaxf(fmaxf(fabsf(a), fabsf(b)), fmaxf(fabsf(c), fabsf(d)));
}
template <int BITS>
Q4_DEVINL float scale_of_f(float absmax) {
    constexpr float qmax = (float)((1 << (BITS - 1)) - 1);
    const float s = __fdiv_rn(absmax, qmax);
    return s == 0.0f ? 1.0f : s;
}

// ---------------------------------------------------------------------------------------
// Coalesced kernel for compile-time groups G in {16, ..., 1024} that divide 1024.
// A warp handles a chunk of 1024 consecutive weights: load u (u = 0..7) of lane l is the
// float4 at 4 * (32 u + l), so every load instruction reads 512 contiguous bytes. A group
// of G <= 128 lies inside one load (G/4 lanes, shuffle reduction); a larger group spans
// G/128 loads of the whole warp. Packed bytes are transposed through shared memory so
// that each lane writes one (int4) or two (int8) 128-bit stores. Registers are capped
// for four CTAs (32 warps) per SM: more chunks in flight per SM to cover the load latency.
template <int BITS, int G>
__global__ void __launch_bounds__(256, 4) qpack_chunk(const float *__restrict__ w, int64_t nchunks,
                                                      uint8_t *__restrict__ payload,
                                                      float *__restrict__ scales,
                                                      uint32_t *__restrict__ status) {
    constexpr int U = 8;                         // float4 loads per lane per chunk
    constexpr int CH = 32 * 4 * U;               // 1024 weights per warp chunk
    constexpr int CB = CH * BITS / 8;            // packed bytes per chunk
    constexpr int LPG = G >= 128 ? 32 : G / 4;   // lanes sharing a group inside one load
    constexpr int UPG = G >= 128 ? G / 128 : 1;  // loads spanned by one group
    __shared__ __align__(16) uint8_t stage[8][CB];
    const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
    uint8_t *my = stage[wib];
    const int64_t warp0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    bool nonfinite = false;
    for (int64_t c = warp0; c < nchunks; c += nwarps) {
        const float *src = w + c * CH;
        float v[U][4];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const float4 f = ld_nc_f4(src + 4 * (32 * u + lane));
            v[u][0] = f.x; v[u][1] = f.y; v[u][2] = f.z; v[u][3] = f.w;
        }
        float m[U];
#pragma unroll
        for (int u = 0; u < U; ++u) m[u] = absmax4(v[u][0], v[u][1], v[u][2], v[u][3]);
#pragma unroll
        for (int u = 0; u < U; u += UPG) {
#pragma unroll
            for (int q = 1; q < UPG; ++q) m[u] = fmaxf(m[u], m[u + q]);
#pragma unroll
            for (int off = 1; off < LPG; off <<= 1) m[u] = fmaxf(m[u], __shfl_xor_sync(0xffffffffu, m[u], off));
        }
        // The scale and reciprocal of each group are computed once, by one lane per
        // group (lane L takes group L, L + 32, ...), and handed back by shuffles; the
        // division and reciprocal are the same IEEE operations whichever lane does them.
        constexpr int NGC = CH / G;                 // groups in the chunk
        constexpr int GPL = G >= 128 ? 1 : 128 / G; // groups per load (when G < 128)
        constexpr int NR = (NGC + 31) / 32;         // groups per lane
        float s_own[NR], r_own[NR];
        bool fast_own[NR];
#pragma unroll
        for (int rr = 0; rr < NR; ++rr) {
            const int gi = lane + 32 * rr;          // the group this lane computes
            const int ug = G >= 128 ? gi * UPG : gi / GPL;  // its first load
            const int lp = G >= 128 ? 0 : (gi % GPL) * LPG; // a lane holding its max
            float mg = 0.f;
#pragma unroll
            for (int u = 0; u < U; u += UPG) {
                const float t = __shfl_sync(0xffffffffu, m[u], lp);
                mg = (u == ug) ? t : mg;
            }
            const float sc = scale_of_f<BITS>(mg);
            const GroupDiv dd = make_div(sc);
            s_own[rr] = sc;
            r_own[rr] = dd.r;
            fast_own[rr] = dd.fast;
            if (gi < NGC) scales[c * NGC + gi] = sc;
        }
#pragma unroll
        for (int u = 0; u < U; u += UPG) {
            // this lane's group in load u, and the lane that computed it
            // (the groups of one load never straddle a multiple of 32, so the register
            // set rr is the same in every lane and in the source lane)
            const int gi = G >= 128 ? u / UPG : u * GPL + lane / LPG;
            const int rr = (G >= 128 ? u / UPG : u * GPL) / 32, src = gi % 32;
            GroupDiv d;
            d.s = __shfl_sync(0xffffffffu, s_own[NR > 1 ? rr : 0], src);
            d.r = __shfl_sync(0xffffffffu, r_own[NR > 1 ? rr : 0], src);
            d.fast = __shfl_sync(0xffffffffu, (int)fast_own[NR > 1 ? rr : 0], src) != 0;
#pragma unroll
            for (int q = 0; q < UPG; ++q) {
                const int uu = u + q;
                uint32_t t[4];
                codes4<BITS>(v[uu], d, t, nonfinite);
                const int e = 32 * uu + lane;  // float4 index inside the chunk
                if constexpr (BITS == 4)
                    reinterpret_cast<uint16_t *>(my)[e] = (uint16_t)pack4<4>(t);
                else
                    reinterpret_cast<uint32_t *>(my)[e] = pack4<8>(t);
            }
        }
        __syncwarp();
        uint8_t *dst = payload + c * CB;
#pragma unroll
        for (int q = 0; q < CB / 512; ++q)
            st_v4(dst + 512 * q + 16 * lane, reinterpret_cast<const uint4 *>(my)[32 * q + lane]);
        __syncwarp();
    }
    if (nonfinite && status) atomicOr(status, Q4_STATUS_NONFINITE);
}

// ---------------------------------------------------------------------------------------
// One CTA of 256 threads per group (large groups, e.g. one scale per output channel).
// Thread t owns float4 number q * 256 + t for q < NQ (coalesced), the group stays in
// registers, the absmax is a block reduction, and codes are stored with 16-bit (int4)
// or 32-bit (int8) coalesced stores.
template <int BITS, int NQ>
__global__ void __launch_bounds__(256) qpack_group_cta(const float *__restrict__ w, int64_t group,
                                                       uint8_t *__restrict__ payload,
                                                       float *__restrict__ scales,
                                                       uint32_t *__restrict__ status) {
    __shared__ float red[8];
    const int tid = threadIdx.x;
    const int64_t gidx = blockIdx.x;
    const int64_t base = gidx * group;
    const int n4 = (int)(group / 4);
    float v[NQ][4];
    float m = 0.f;
#pragma unroll
    for (int q = 0; q < NQ; ++q) {
        const int idx = q * 256 + tid;
        if (idx < n4) {
            const float4 f = ld_nc_f4(w + base + 4 * (int64_t)idx);
            v[q][0] = f.x; v[q][1] = f.y; v[q][2] = f.z; v[q][3] = f.w;
            m = fmaxf(m, absmax4(f.x, f.y, f.z, f.w));
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    if ((tid & 31) == 0) red[tid >> 5] = m;
    __syncthreads();
    m = red[0];
#pragma unroll
    for (int i = 1; i < 8; ++i) m = fmaxf(m, red[i]);
    const float s = scale_of_f<BITS>(m);
    if (tid == 0) scales[gidx] = s;
    const GroupDiv d = make_div(s);
    bool nonfinite = false;
#pragma unroll
    for (int q = 0; q < NQ; ++q) {
        const int idx = q * 256 + tid;
        if (idx < n4) {
            uint32_t t[4];
            codes4<BITS>(v[q], d, t, nonfinite);
            const int64_t e = base + 4 * (int64_t)idx;
            if constexpr (BITS == 4)
                *reinterpret_cast<uint16_t *>(payload + e / 2) = (uint16_t)pack4<4>(t);
            else
                *reinterpret_cast<uint32_t *>(payload + e) = pack4<8>(t);
        }
    }
    if (nonfinite && status) atomicOr(status, Q4_STATUS_NONFINITE);
}

// ---------------------------------------------------------------------------------------
// Generic path: groups [g0, g1), one warp per group.
template <int BITS>
__global__ void __launch_bounds__(256) qpack_generic_scales(const float *__restrict__ w,
                                                            int64_t group, int64_t g0, int64_t g1,
                                                            float *__restrict__ scales,
                                                            uint32_t *__restrict__ status) {
    const int lane = threadIdx.x & 31;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t gi = g0 + (((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5); gi < g1;
         gi += nwarps) {
        uint32_t m = 0;
        const float *p = w + gi * group;
        for (int64_t i = lane; i < group; i += 32) m = max(m, absbits(p[i]));
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, off));
        if (lane == 0) {
            scales[gi] = scale_of<BITS>(m);
            if (m >= kInfBits && status) atomicOr(status, Q4_STATUS_NONFINITE);
        }
    }
}

// Output bytes [b0, b1): int4 byte t holds weights 2t and 2t+1 (possibly of two groups).
template <int BITS>
__global__ void __launch_bounds__(256) qpack_generic_codes(const float *__restrict__ w,
                                                           int64_t group, int64_t b0, int64_t b1,
                                                           const float *__restrict__ scales,
                                                           uint8_t *__restrict__ payload) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t b = b0 + (int64_t)blockIdx.x * blockDim.x + threadIdx.x; b < b1; b += stride) {
        if constexpr (BITS == 8) {
            payload[b] = (uint8_t)(code_of<8>(w[b], scales[b / group]) & 0xff);
        } else {
            const int64_t e = 2 * b;
            const int lo = code_of<4>(w[e], scales[e / group]) + 8;
            const int hi = code_of<4>(w[e + 1], scales[(e + 1) / group]) + 8;
            payload[b] = (uint8_t)(lo | (hi << 4));
        }
    }
}

// ---------------------------------------------------------------------------------------
// Dequantize 8 weights per thread when g % 8 == 0 (all 8 share one scale).
template <int BITS>
__global__ void __launch_bounds__(256) qdequant_vec(const uint8_t *__restrict__ payload,
                                                    const float *__restrict__ scales,
                                                    int64_t n8, int64_t group,
                                                    float *__restrict__ out) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n8; i += stride) {
        const int64_t e = 8 * i;
        const float s = scales[e / group];
        float r[8];
        if constexpr (BITS == 4) {
            const uint32_t word = *reinterpret_cast<const uint32_t *>(payload + 4 * i);
#pragma unroll
            for (int j = 0; j < 8; ++j) r[j] = __fmul_rn((float)((int)((word >> (4 * j)) & 15u) - 8), s);
        } else {
            const uint2 q = *reinterpret_cast<const uint2 *>(payload + 8 * i);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                r[j] = __fmul_rn((float)(int8_t)(q.x >> (8 * j)), s);
                r[4 + j] = __fmul_rn((float)(int8_t)(q.y >> (8 * j)), s);
            }
        }
        float4 *o = reinterpret_cast<float4 *>(out + e);
        o[0] = make_float4(r[0], r[1], r[2], r[3]);
        o[1] = make_float4(r[4], r[5], r[6], r[7]);
    }
}

template <int BITS>
__global__ void __launch_bounds__(256) qdequant_generic(const uint8_t *__restrict__ payload,
                                                        const float *__restrict__ scales,
                                                        int64_t n, int64_t group,
                                                        float *__restrict__ out) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += stride) {
        int c;
        if constexpr (BITS == 8) {
            c = (int8_t)payload[e];
        } else {
            const uint32_t b = payload[e >> 1];
            c = (int)((e & 1) ? (b >> 4) : (b & 15u)) - 8;
        }
        out[e] = __fmul_rn((float)c, scales[e / group]);
    }
}

inline int grid_for(int64_t work, int per_block, int max_blocks) {
    int64_t b = (work + per_block - 1) / per_block;
    if (b < 1) b = 1;
    return (int)(b < max_blocks ? b : max_blocks);
}

template <int BITS>
cudaError_t launch_qpack_bits(const float *w, int64_t n, int64_t group, uint8_t *payload,
                              float *scales, uint32_t *status, cudaStream_t st, int sms) {
    const bool aligned = ((uintptr_t)w % 16 == 0) && ((uintptr_t)payload % 16 == 0);
    int64_t done_groups = 0;  // groups [0, done_groups) handled by a vector kernel
    if (aligned && group >= 16 && group <= 1024 && 1024 % group == 0 && n >= 1024) {
        const int64_t nchunks = n / 1024;
        const int blocks = grid_for(nchunks * 32, 256, sms * 8);
#define Q4_CHUNK(G)                                                                          \
    case G:                                                                                  \
        qpack_chunk<BITS, G><<<blocks, 256, 0, st>>>(w, nchunks, payload, scales, status);   \
        break;
        switch ((int)group) {
            Q4_CHUNK(16) Q4_CHUNK(32) Q4_CHUNK(64) Q4_CHUNK(128) Q4_CHUNK(256) Q4_CHUNK(512) Q4_CHUNK(1024)
            default: return cudaErrorInvalidValue;
        }
#undef Q4_CHUNK
        done_groups = nchunks * 1024 / group;
    } else if (aligned && group % 4 == 0 && group > 1024 && group <= 32 * 1024) {
        const int64_t ngroups = n / group;
        const int64_t nq = (group / 4 + 255) / 256;
        const unsigned gb = (unsigned)ngroups;  // grid.x limit 2^31-1: far above any real count
        if (nq <= 1) qpack_group_cta<BITS, 1><<<gb, 256, 0, st>>>(w, group, payload, scales, status);
        else if (nq <= 2) qpack_group_cta<BITS, 2><<<gb, 256, 0, st>>>(w, group, payload, scales, status);
        else if (nq <= 4) qpack_group_cta<BITS, 4><<<gb, 256, 0, st>>>(w, group, payload, scales, status);
        else if (nq <= 8) qpack_group_cta<BITS, 8><<<gb, 256, 0, st>>>(w, group, payload, scales, status);
        else if (nq <= 16) qpack_group_cta<BITS, 16><<<gb, 256, 0, st>>>(w, group, payload, scales, status);
        else qpack_group_cta<BITS, 32><<<gb, 256, 0, st>>>(w, group, payload, scales, status);
        done_groups = ngroups;
    }
    const int64_t ngroups = n / group;
    if (done_groups < ngroups) {
        const int64_t g0 = done_groups;
        qpack_generic_scales<BITS><<<grid_for((ngroups - g0) * 32, 256, sms * 8), 256, 0, st>>>(
            w, group, g0, ngroups, scales, status);
        const int64_t e0 = g0 * group;  // first weight not yet packed (even: vector kernels
                                        // only take groups that are multiples of 16)
        const int64_t b0 = (BITS == 4) ? e0 / 2 : e0;
        const int64_t b1 = (BITS == 4) ? n / 2 : n;
        qpack_generic_codes<BITS><<<grid_for(b1 - b0, 256, sms * 16), 256, 0, st>>>(
            w, group, b0, b1, scales, payload);
    }
    return cudaGetLastError();
}

template <int BITS>
cudaError_t launch_qdequant_bits(const uint8_t *payload, const float *scales, int64_t n,
                                 int64_t group, float *out, cudaStream_t st, int sms) {
    const bool aligned = ((uintptr_t)payload % 8 == 0) && ((uintptr_t)out % 16 == 0);
    if (aligned && group % 8 == 0 && n % 8 == 0) {
        const int64_t n8 = n / 8;
        qdequant_vec<BITS><<<grid_for(n8, 256, sms * 16), 256, 0, st>>>(payload, scales, n8, group, out);
    } else {
        qdequant_generic<BITS><<<grid_for(n, 256, sms * 16), 256, 0, st>>>(payload, scales, n, group, out);
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_qpack(const float *w, int64_t n, int bits, int64_t group, uint8_t *payload,
                         float *scales, uint32_t *status, cudaStream_t st, int sms) {
    return bits == 4 ? launch_qpack_bits<4>(w, n, group, payload, scales, status, st, sms)
                     : launch_qpack_bits<8>(w, n, group, payload, scales, status, st, sms);
}

cudaError_t launch_qdequant(const uint8_t *payload, const float *scales, int64_t n, int bits,
                            int64_t group, float *out, cudaStream_t st, int sms) {
    return bits == 4 ? launch_qdequant_bits<4>(payload, scales, n, group, out, st, sms)
                     : launch_qdequant_bits<8>(payload, scales, n, group, out, st, sms);
}

}  // namespace q4
