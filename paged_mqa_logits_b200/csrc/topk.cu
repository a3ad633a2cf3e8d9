// Top-k selection over the logits: the indexer's use of them (the page
// "[flashinfer] Blackwell 아키텍처를 위한 고성능 Paged MQA Logits 커널 도입",
// introduction: the DeepSeek sparse-attention indexer scores every cached
// token and sparse attention then reads the best-scoring ones).
//
// For every row (b, n): the k tokens t < ctx_{b,n} of largest logit, ordered
// by logit descending and, for equal logits, by token ascending (-0.0 and
// +0.0 are equal); rows with fewer than k valid tokens are padded with -1.
//
// One CTA per row. Logits map to order-preserving 32-bit keys. A radix select
// (three passes of 11 / 11 / 10 bits, histograms in shared memory, a block
// suffix scan to pick the digit) finds the k-th largest key T and how many
// tokens equal to T to take; one pass in token order then takes every key > T
// and the first keys == T (block prefix sums keep token order); a bitonic sort
// of the (key, token) pairs in shared memory orders the result.
#include <cuda_runtime.h>

#include <cstdint>

#include "mqa_logits.h"

namespace mqa {

constexpr int kTopkThreads = 1024;
constexpr int kTopkBins = 2048;  // widest radix digit: 11 bits

// Order-preserving map of fp32 to uint32 (larger value, larger key); -0.0
// maps like +0.0.
__device__ __forceinline__ uint32_t topk_key(float v) {
    uint32_t u = __float_as_uint(v);
    if (u == 0x80000000u) u = 0u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Block-wide exclusive prefix sum of v over the CTA's threads (in thread
// order); `total` gets the sum. Uses ws[0..32] of shared memory.
__device__ __forceinline__ int block_exscan(int v, int* ws, int& total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int x = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += x;
    }
    if (lane == 31) ws[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int w = lane < nw ? ws[lane] : 0;
        int wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int x = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o) wi += x;
        }
        if (lane < nw) ws[lane] = wi - w;
        if (lane == 31) ws[32] = wi;
    }
    __syncthreads();
    const int ex = ws[warp] + incl - v;
    total = ws[32];
    __syncthreads();  // ws is reused by the next call
    return ex;
}

__global__ void __launch_bounds__(kTopkThreads)
topk_kernel(const float* __restrict__ logits, const int32_t* __restrict__ context_lens,
            int next_n, int L, int k, int sort_n, int32_t* __restrict__ out) {
    extern __shared__ uint64_t sel[];                 // [sort_n] (key << 32) | ~token
    __shared__ int hist[kTopkBins];
    __shared__ int ws[33];
    __shared__ int bcast[2];

    const int row = blockIdx.x;
    const int b = row / next_n, n = row - b * next_n;
    int c = __ldg(context_lens + b);
    c = c < 0 ? 0 : (c > L ? L : c);
    int cbn = c - next_n + 1 + n;
    cbn = cbn < 0 ? 0 : (cbn > c ? c : cbn);
    const float* x = logits + (int64_t)row * L;
    const int m = cbn < k ? cbn : k;                  // tokens taken
    const int tid = threadIdx.x, nthr = blockDim.x;

    uint32_t T = 0;       // keys > T are all taken
    int take_eq = 0;      // ... and the first take_eq keys == T, in token order
    if (cbn > k) {
        uint32_t prefix = 0, mask = 0;
        int remaining = k;  // still to take among keys matching `prefix`
#pragma unroll
        for (int p = 0; p < 3; ++p) {
            const int sh = p == 0 ? 21 : (p == 1 ? 10 : 0);  // digits: bits 31-21, 20-10, 9-0
            const int nb = p == 2 ? 1024 : 2048;
            for (int i = tid; i < nb; i += nthr) hist[i] = 0;
            __syncthreads();
            for (int t = tid; t < cbn; t += nthr) {
                const uint32_t key = topk_key(__ldg(x + t));
                if ((key & mask) == prefix) atomicAdd(&hist[(key >> sh) & (nb - 1)], 1);
            }
            __syncthreads();
            // digit d: (count of digits > d) < remaining <= (count of digits >= d).
            // Thread i owns digits nb-1-2i and nb-2-2i (top down), so a prefix sum
            // over threads is a suffix sum over digits.
            const int d0 = nb - 1 - 2 * tid, d1 = d0 - 1;
            const int h0 = d0 >= 0 ? hist[d0] : 0, h1 = d1 >= 0 ? hist[d1] : 0;
            int total;
            const int above = block_exscan(h0 + h1, ws, total);  // digits > d0
            if (d0 >= 0 && above < remaining && remaining <= above + h0) {
                bcast[0] = d0;
                bcast[1] = remaining - above;
            } else if (d1 >= 0 && above + h0 < remaining && remaining <= above + h0 + h1) {
                bcast[0] = d1;
                bcast[1] = remaining - above - h0;
            }
            __syncthreads();
            prefix |= (uint32_t)bcast[0] << sh;
            mask |= (uint32_t)(nb - 1) << sh;
            remaining = bcast[1];
            __syncthreads();
        }
        T = prefix;
        take_eq = remaining;
    }

    // Take, in token order: every key > T, and keys == T while fewer than
    // take_eq of them were taken (with cbn <= k every valid token is taken).
    int base_eq = 0, base_sel = 0;
    for (int start = 0; start < cbn; start += nthr) {
        const int t = start + tid;
        const uint32_t key = t < cbn ? topk_key(__ldg(x + t)) : 0u;
        const bool all = cbn <= k;
        const bool gt = t < cbn && (all || key > T);
        const bool eq = t < cbn && !all && key == T;
        int neq, nsel;
        const int rank_eq = base_eq + block_exscan(eq ? 1 : 0, ws, neq);
        const bool take = gt || (eq && rank_eq < take_eq);
        const int pos = base_sel + block_exscan(take ? 1 : 0, ws, nsel);
        if (take) sel[pos] = ((uint64_t)key << 32) | (uint32_t)(~(uint32_t)t);
        base_eq += neq;
        base_sel += nsel;
    }
    for (int i = m + tid; i < sort_n; i += nthr) sel[i] = 0ull;  // sorts last
    __syncthreads();

    // bitonic sort, descending: key descending, then token ascending
    for (int size = 2; size <= sort_n; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            for (int i = tid; i < (sort_n >> 1); i += nthr) {
                const int lo = 2 * i - (i & (stride - 1));
                const int hi = lo + stride;
                const uint64_t a = sel[lo], bb = sel[hi];
                const bool desc = (lo & size) == 0;
                if (desc ? (a < bb) : (a > bb)) {
                    sel[lo] = bb;
                    sel[hi] = a;
                }
            }
            __syncthreads();
        }
    }

    int32_t* o = out + (int64_t)row * k;
    for (int i = tid; i < k; i += nthr)
        o[i] = i < m ? (int32_t)(~(uint32_t)(sel[i] & 0xffffffffull)) : -1;
}

// Host launcher: one CTA per row; sort_n = next power of two >= k.
int launch_topk(const float* logits, const int32_t* context_lens, int batch, int next_n, int L,
                int k, int32_t* out, void* stream) {
    int sort_n = 1;
    while (sort_n < k) sort_n <<= 1;
    if (sort_n < 2) sort_n = 2;
    const size_t smem = (size_t)sort_n * 8;
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, topk_kernel);
    if (e != cudaSuccess) return (int)e;
    if (fa.maxDynamicSharedSizeBytes < (int)smem) {
        e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smem);
        if (e != cudaSuccess) return (int)e;
    }
    topk_kernel<<<batch * next_n, kTopkThreads, smem, static_cast<cudaStream_t>(stream)>>>(
        logits, context_lens, next_n, L, k, sort_n, out);
    return (int)cudaGetLastError();
}

}  // namespace mqa
