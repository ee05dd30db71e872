// anygroup.cu -- qgemm for every group size the format allows.
//
// pack() on the "量化推理：INT8/INT4 的体积、困惑度与速度为什么不同步" page reshapes the whole
// flattened tensor to (-1, group): a group may be any divisor of N * K, so it can cross
// rows at a different offset in every row (g = 3K/2), or be narrower than the GEMV's
// 32-wide segments (g = 16, g = 48), and an int4 row of odd K starts in the middle of a
// byte. The fused GEMV and the tensor-core GEMM take the regular groups (dividing K in
// multiples of 32, or whole rows); this kernel takes the rest.
//
// One warp computes y[m][n] for one weight row n and up to eight rows of x. Each lane
// takes eight consecutive weights at a time (k = 8 * lane + 256 * j; up to four such
// chunks in flight when x has one or two rows). It decodes their codes from the
// flattened payload (element e = n * K + k; int4: nibble e & 1 of byte e / 2, code =
// nibble - 8; int8: the byte as a signed value), forms w' = fl32(code * scale[e / group])
// exactly as qdequant does. The eight products w' * x of a chunk go into one fp32 fma
// chain (each product exact inside its fma), and the chunk sums into a compensated
// (Kahan) fp32 sum; the lanes' sums meet in a fixed shuffle tree. The chain rounds at most
// eight times, the compensated sum about twice and the tree five times, so
// |y - sum_k w'x| <= 2^-20 * sum_k |w'x|, far inside qgemm's 1e-5.
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include <cstdint>

#include "kernels.h"

namespace q4 {
namespace {

constexpr int kAnyWarps = 8;   // warps per CTA
constexpr int kAnyRows = 8;    // rows of x per warp

// The codes of elements e .. e + 7 as 8 unsigned fields (bytes past the payload's nbytes
// read as zero): int4, 8 nibbles (code + 8) in lo, element e lowest; int8, 8 bytes (code
// as two's complement) in lo (e .. e + 3) and hi. pal: the payload is 4-byte aligned, so
// whole words can be read.
template <int BITS>
__device__ __forceinline__ void codes8_at(const uint8_t *__restrict__ payload, int64_t nbytes, bool pal, int64_t e,
                                          uint32_t &lo, uint32_t &hi) {
    if (BITS == 4) {
        const int64_t b = e >> 1;                 // first byte
        const int64_t a = b & ~(int64_t)3;        // its 4-byte word
        uint32_t w0 = 0, w1 = 0;
        if (pal && a + 8 <= nbytes) {
            w0 = __ldg(reinterpret_cast<const uint32_t *>(payload + a));
            w1 = __ldg(reinterpret_cast<const uint32_t *>(payload + a + 4));
        } else {
            for (int i = 0; i < 4 && a + i < nbytes; ++i) w0 |= (uint32_t)__ldg(payload + a + i) << (8 * i);
            for (int i = 0; i < 4 && a + 4 + i < nbytes; ++i) w1 |= (uint32_t)__ldg(payload + a + 4 + i) << (8 * i);
        }
        const uint32_t sh = (uint32_t)(8 * (b - a) + 4 * (e & 1));  // bit of element e's nibble, < 32
        lo = (uint32_t)(((uint64_t)w1 << 32 | w0) >> sh);
        hi = 0;
    } else {
        const int64_t a = e & ~(int64_t)3;
        uint32_t w[3];
        if (pal && a + 12 <= nbytes) {
#pragma unroll
            for (int i = 0; i < 3; ++i) w[i] = __ldg(reinterpret_cast<const uint32_t *>(payload + a + 4 * i));
        } else {
#pragma unroll
            for (int i = 0; i < 3; ++i) {
                w[i] = 0;
                for (int j = 0; j < 4; ++j)
                    if (a + 4 * i + j < nbytes) w[i] |= (uint32_t)__ldg(payload + a + 4 * i + j) << (8 * j);
            }
        }
        const uint32_t sh = (uint32_t)(8 * (e - a));
        lo = __funnelshift_r(w[0], w[1], sh);
        hi = __funnelshift_r(w[1], w[2], sh);
    }
}

// Code i of the eight as an exact float: the field ORed into the mantissa of 2^23, minus
// 2^23 and the field's offset (8 for int4 nibbles; int8 bytes have their sign bit flipped
// first, offset 128).
template <int BITS>
__device__ __forceinline__ float code_f(uint32_t lo, uint32_t hi, int i) {
    if (BITS == 4) {
        const uint32_t f = (lo >> (4 * i)) & 15u;
        return __fsub_rn(__uint_as_float(0x4B000000u | f), 8388616.0f);
    } else {
        const uint32_t f = (((i < 4 ? lo : hi) >> (8 * (i & 3))) & 255u) ^ 128u;
        return __fsub_rn(__uint_as_float(0x4B000000u | f), 8388736.0f);
    }
}

// x[i .. i + 7] (zeros past cnt), as 16-byte loads when row and element line up.
template <bool XBF16>
__device__ __forceinline__ void x8_at(const void *x, int64_t i, int cnt, bool vec, float (&v)[8]) {
    if (XBF16) {
        const __nv_bfloat16 *p = reinterpret_cast<const __nv_bfloat16 *>(x) + i;
        if (vec && cnt == 8) {
            const uint4 u = __ldg(reinterpret_cast<const uint4 *>(p));
            const uint32_t ww[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                v[2 * q] = __uint_as_float(ww[q] << 16);
                v[2 * q + 1] = __uint_as_float(ww[q] & 0xffff0000u);
            }
        } else {
#pragma unroll
            for (int q = 0; q < 8; ++q) v[q] = q < cnt ? __bfloat162float(p[q]) : 0.f;
        }
    } else {
        const float *p = reinterpret_cast<const float *>(x) + i;
        if (vec && cnt == 8) {
            const float4 a = __ldg(reinterpret_cast<const float4 *>(p));
            const float4 b = __ldg(reinterpret_cast<const float4 *>(p) + 1);
            v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
            v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
        } else {
#pragma unroll
            for (int q = 0; q < 8; ++q) v[q] = q < cnt ? __ldg(p + q) : 0.f;
        }
    }
}

// e / group for 0 <= e < 2^40, from a double reciprocal, corrected to the exact quotient.
__device__ __forceinline__ int64_t div_group(int64_t e, int64_t group, double inv) {
    int64_t q = (int64_t)((double)e * inv);
    int64_t r = e - q * group;
    if (r < 0) {
        --q;
        r += group;
    }
    if (r >= group) ++q;
    return q;
}

// One warp per weight row n and chunk of up to kAnyRows rows of x (grid: rows of W by
// chunks of x); UNR chunks of eight weights per lane have their codes and scales in flight
// at once.
template <int BITS, bool XBF16, int UNR, int MR>
__global__ void __launch_bounds__(32 * kAnyWarps) qgemm_any_group(const void *__restrict__ x, int64_t M,
                                                                 const uint8_t *__restrict__ payload,
                                                                 const float *__restrict__ scales, int64_t N,
                                                                 int64_t K, int64_t group, double inv_group,
                                                                 float *__restrict__ y) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t nbytes = (N * K * BITS + 7) / 8;
    const bool pal = (uintptr_t)payload % 4 == 0;
    // 16-byte loads of x when every row and every lane's first element line up
    const bool xvec = ((uintptr_t)x % 16 == 0) && (K % (XBF16 ? 8 : 4) == 0);
    for (int64_t mb = blockIdx.y; mb * MR < M; mb += gridDim.y)
    for (int64_t n = (int64_t)blockIdx.x * kAnyWarps + warp; n < N; n += (int64_t)gridDim.x * kAnyWarps) {
        const int64_t m0 = mb * MR;
        const int mc = (int)(M - m0 < MR ? M - m0 : MR);
        float sum[MR], cmp[MR];  // compensated sums of the chunk sums
#pragma unroll
        for (int m = 0; m < MR; ++m) sum[m] = cmp[m] = 0.f;
        int64_t e = n * K + 8 * (int64_t)lane;  // first element of this lane's next eight
        int64_t q = div_group(e, group, inv_group), r = e - q * group;
        for (int64_t k0 = 8 * (int64_t)lane; k0 < K; k0 += 256 * UNR) {
            // codes and scales of UNR chunks (independent loads); element i of a chunk is in
            // group q + (r + i) / group, r being element e's place in group q
            uint32_t clo[UNR], chi[UNR];
            float s0[UNR], s1[UNR];
            int bnd[UNR], cnt[UNR];
#pragma unroll
            for (int j = 0; j < UNR; ++j) {
                const int64_t kj = k0 + 256 * j;
                cnt[j] = kj < K ? (int)(K - kj < 8 ? K - kj : 8) : 0;
                codes8_at<BITS>(payload, nbytes, pal, cnt[j] ? e : 0, clo[j], chi[j]);
                bnd[j] = (int)(group - r < 8 ? group - r : 8);  // first element of the next group
                s0[j] = cnt[j] ? __ldg(scales + q) : 0.f;
                s1[j] = cnt[j] && bnd[j] < cnt[j] && group >= 8 ? __ldg(scales + q + 1) : s0[j];
                e += 256;
                r += 256;
                if (r >= group) {
                    if (group >= 256) {
                        r -= group;
                        ++q;
                    } else {  // r < 512
                        q += (int)r / (int)group;
                        r = (int)r % (int)group;
                    }
                }
            }
#pragma unroll
            for (int j = 0; j < UNR; ++j) {
                if (!cnt[j]) continue;
                float w[8];
                if (group >= 8) {
#pragma unroll
                    for (int i = 0; i < 8; ++i) w[i] = __fmul_rn(code_f<BITS>(clo[j], chi[j], i), i < bnd[j] ? s0[j] : s1[j]);
                } else {  // narrow groups: every element may need its own scale
                    const int64_t ej = e - 256 * (UNR - j);
                    const int64_t qj = div_group(ej, group, inv_group);
                    const int rj = (int)(ej - qj * group);
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        w[i] = i < cnt[j] ? __fmul_rn(code_f<BITS>(clo[j], chi[j], i), __ldg(scales + qj + (rj + i) / (int)group))
                                          : 0.f;
                }
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    if (i >= cnt[j]) w[i] = 0.f;
#pragma unroll
                for (int m = 0; m < MR; ++m) {
                    if (m < mc) {
                        float xv[8];
                        x8_at<XBF16>(x, (m0 + m) * K + k0 + 256 * j, cnt[j], xvec, xv);
                        // the chunk's sum: exact-product fma chain, then a compensated add
                        float cs = __fmul_rn(w[0], xv[0]);
#pragma unroll
                        for (int i = 1; i < 8; ++i) cs = __fmaf_rn(w[i], xv[i], cs);
                        const float t = __fsub_rn(cs, cmp[m]);
                        const float s2 = __fadd_rn(sum[m], t);
                        cmp[m] = __fsub_rn(__fsub_rn(s2, sum[m]), t);
                        sum[m] = s2;
                    }
                }
            }
        }
        // the lanes' sums in a fixed shuffle tree
#pragma unroll
        for (int m = 0; m < MR; ++m) {
            float v = __fsub_rn(sum[m], cmp[m]);
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1) v = __fadd_rn(v, __shfl_xor_sync(0xffffffffu, v, off));
            if (lane == 0 && m < mc) y[(m0 + m) * N + n] = v;
        }
    }
}

template <int BITS, bool XBF16>
cudaError_t any_group_go(const void *x, int64_t M, const uint8_t *payload, const float *scales, int64_t N, int64_t K,
                         int64_t group, float *y, int sms, cudaStream_t st) {
    const int64_t want = (N + kAnyWarps - 1) / kAnyWarps;
    const int64_t cap = (int64_t)(sms > 0 ? sms : 148) * 8;
    const unsigned gx = (unsigned)(want < cap ? want : cap);
    const double inv = 1.0 / (double)group;
    auto gy = [&](int mr) { const int64_t c = (M + mr - 1) / mr; return (unsigned)(c < 65535 ? c : 65535); };
    const dim3 block(32 * kAnyWarps);
    if (M <= 1)
        qgemm_any_group<BITS, XBF16, 4, 1><<<dim3(gx, gy(1)), block, 0, st>>>(x, M, payload, scales, N, K, group, inv, y);
    else if (M <= 2)
        qgemm_any_group<BITS, XBF16, 2, 2><<<dim3(gx, gy(2)), block, 0, st>>>(x, M, payload, scales, N, K, group, inv, y);
    else
        qgemm_any_group<BITS, XBF16, 1, kAnyRows><<<dim3(gx, gy(kAnyRows)), block, 0, st>>>(x, M, payload, scales, N, K,
                                                                                        group, inv, y);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_any_group(const void *x, bool x_bf16, int64_t M, const uint8_t *payload, const float *scales,
                             int64_t N, int64_t K, int bits, int64_t group, float *y, int sms, cudaStream_t st) {
    if (M <= 0 || N <= 0) return cudaSuccess;
    if (bits == 4)
        return x_bf16 ? any_group_go<4, true>(x, M, payload, scales, N, K, group, y, sms, st)
                      : any_group_go<4, false>(x, M, payload, scales, N, K, group, y, sms, st);
    return x_bf16 ? any_group_go<8, true>(x, M, payload, scales, N, K, group, y, sms, st)
                  : any_group_go<8, false>(x, M, payload, scales, N, K, group, y, sms, st);
}

}  // namespace q4
