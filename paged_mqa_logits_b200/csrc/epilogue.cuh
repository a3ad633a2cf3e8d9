// The logits epilogue shared by the FP8 and FP4 kernels: one thread per token
// (its TMEM lane) reads the token's H*next_n accumulator columns and forms,
// per draft row n,
//   logit = post * sum_h w[n,h] * max(scale * acc[nH + h], 0)
// then writes it, or -inf at and past the draft row's context (a select, so
// stale data past the context can never leak into the output).
#pragma once
#include <cstdint>
#include "ptx.cuh"

namespace mqa {

// Four interleaved partial sums (heads h = 4i + j go to partial j), so the
// fused multiply-adds form four short dependency chains instead of one long
// one; acc[] carries the partials across chunks of heads. The token's scale
// s is applied outside the sum, which is the same value:
// w * max(s * v, 0) = s * (w * max(v, 0)) for s >= 0, and
// w * max(s * v, 0) = s * (w * min(v, 0)) for s < 0 (`neg`).
// The multiply-adds go two at a time (fma.rn.f32x2: partials 0/1 and 2/3),
// each half the same fp32 fused multiply-add as fmaf.
template <int N>
__device__ __forceinline__ void head_sum(const float (&v)[N], const float* w, bool neg,
                                         float (&acc)[4]) {
    uint64_t a01 = ptx::f32x2_pack(acc[0], acc[1]), a23 = ptx::f32x2_pack(acc[2], acc[3]);
#pragma unroll
    for (int h = 0; h < N; h += 4) {
        const float4 w4 = *reinterpret_cast<const float4*>(w + h);
        float r0, r1, r2, r3;
        if (!neg) {
            r0 = fmaxf(v[h + 0], 0.f), r1 = fmaxf(v[h + 1], 0.f);
            r2 = fmaxf(v[h + 2], 0.f), r3 = fmaxf(v[h + 3], 0.f);
        } else {
            r0 = fminf(v[h + 0], 0.f), r1 = fminf(v[h + 1], 0.f);
            r2 = fminf(v[h + 2], 0.f), r3 = fminf(v[h + 3], 0.f);
        }
        a01 = ptx::fma_f32x2(ptx::f32x2_pack(w4.x, w4.y), ptx::f32x2_pack(r0, r1), a01);
        a23 = ptx::fma_f32x2(ptx::f32x2_pack(w4.z, w4.w), ptx::f32x2_pack(r2, r3), a23);
    }
    ptx::f32x2_unpack(a01, acc[0], acc[1]);
    ptx::f32x2_unpack(a23, acc[2], acc[3]);
}

// The H (16, 32, 64 or 128) accumulator columns at tacc into v, waited for.
template <int H>
__device__ __forceinline__ void tmem_row(uint32_t tacc, float (&v)[H]) {
    if constexpr (H == 16) {
        ptx::tmem_ld16(tacc, v);
    } else {
#pragma unroll
        for (int x = 0; x < H; x += 32)
            ptx::tmem_ld32(tacc + x, *reinterpret_cast<float(*)[32]>(v + x));
    }
    ptx::tmem_ld_wait();
}

// head_sum's min() form for the rare negative scale. The weights are read
// through volatile loads so that the compiler cannot keep the main sum's
// weight registers alive across both sums.
template <int N>
__device__ __forceinline__ void head_sum_min(const float (&v)[N], const float* w, float (&acc)[4]) {
    const volatile float* wv = w;
#pragma unroll
    for (int h = 0; h < N; h += 4) {
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[j] = fmaf(wv[h + j], fminf(v[h + j], 0.f), acc[j]);
    }
}

// tacc: TMEM address of this warp's lane quarter at the accumulator's first
// column. orow: out + (b * next_n) * L + t. `scale` multiplies every score
// (the token's K scale times any power-of-two pre-scale; it is applied once,
// outside the head sum). The accumulator is released (one arrive per warp on
// acc_empty) as soon as its last columns are in registers.
// kCols: accumulator columns read per TMEM round trip (32-column loads issued
// back to back, then one wait): 64 where the register budget allows it.
template <int H, int kCols = 32>
__device__ __forceinline__ void epilogue_tile(uint32_t tacc, const float* w, float scale,
                                              int nn, int ctx, int t, int L, float* orow,
                                              uint64_t* acc_empty, int lane) {
    const float ninf = __int_as_float(0xff800000);
    const bool in_row = t < L;
    const bool neg = scale < 0.f;
    if constexpr (H < 16) {
        // every draft row fits in the first 32 columns
        float v[32];
        ptx::tmem_ld32(tacc, v);
        ptx::tmem_ld_wait();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(acc_empty);
#pragma unroll
        for (int n = 0; n < 4; ++n) {
            if (n < nn) {
                float sum = 0.f;
#pragma unroll
                for (int h = 0; h < H; ++h) {
                    const float x = neg ? fminf(v[n * H + h], 0.f) : fmaxf(v[n * H + h], 0.f);
                    sum = fmaf(w[n * H + h], x, sum);
                }
                const int cbn = min(max(ctx - nn + 1 + n, 0), ctx);
                if (in_row) orow[(int64_t)n * L] = (t < cbn) ? sum * scale : ninf;
            }
        }
    } else if constexpr (H <= kCols) {
        // One TMEM round trip per draft row. The head sum assumes scale >= 0, so
        // `scale` (a global load issued just before the tile) is needed only
        // after it; a warp with a negative scale on some lane reads the columns
        // again (the accumulator is released only after that) and those lanes
        // take the min() sum.
        for (int n = 0; n < nn; ++n) {
            float v[H];
            tmem_row<H>(tacc + n * H, v);
            float part[4] = {0.f, 0.f, 0.f, 0.f};
            head_sum<H>(v, w + n * H, false, part);
            float sum = (part[0] + part[1]) + (part[2] + part[3]);
            const bool neg_lane = scale < 0.f;
            if (__any_sync(0xffffffffu, neg_lane)) {
                tmem_row<H>(tacc + n * H, v);
                if (neg_lane) {
                    float np[4] = {0.f, 0.f, 0.f, 0.f};
                    head_sum_min<H>(v, w + n * H, np);
                    sum = (np[0] + np[1]) + (np[2] + np[3]);
                }
            }
            if (n == nn - 1) {
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(acc_empty);
            }
            const int cbn = min(max(ctx - nn + 1 + n, 0), ctx);
            if (in_row) orow[(int64_t)n * L] = (t < cbn) ? sum * scale : ninf;
        }
    } else {
        constexpr int kChunk = kCols;
        for (int n = 0; n < nn; ++n) {
            float part[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int c0 = 0; c0 < H; c0 += kChunk) {
                float v[kChunk];
                if constexpr (kChunk == 16) {
                    ptx::tmem_ld16(tacc + n * H + c0, *reinterpret_cast<float(*)[16]>(v));
                } else {
#pragma unroll
                    for (int x = 0; x < kChunk; x += 32)
                        ptx::tmem_ld32(tacc + n * H + c0 + x,
                                       *reinterpret_cast<float(*)[32]>(v + x));
                }
                ptx::tmem_ld_wait();
                if (n == nn - 1 && c0 + kChunk >= H) {
                    ptx::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(acc_empty);
                }
                head_sum<kChunk>(v, w + n * H + c0, neg, part);
            }
            const float sum = (part[0] + part[1]) + (part[2] + part[3]);
            const int cbn = min(max(ctx - nn + 1 + n, 0), ctx);
            if (in_row) orow[(int64_t)n * L] = (t < cbn) ? sum * scale : ninf;
        }
    }
}

}  // namespace mqa
