// Top-k selection over the logits: the indexer's use of them (the page
// "[flashinfer] Blackwell 아키텍처를 위한 고성능 Paged MQA Logits 커널 도입",
// introduction: the DeepSeek sparse-attention indexer scores every cached
// token and sparse attention then reads the best-scoring ones).
//
// For every row (b, n): the k tokens t < ctx_{b,n} of largest logit, ordered
// by logit descending and, for equal logits, by token ascending (-0.0 and
// +0.0 are equal); rows with fewer than k valid tokens are padded with -1.
//
// One CTA per row. Logits map to order-preserving 32-bit keys, cached in
// shared memory when the row's valid part fits. A radix select (three passes
// of 11 / 11 / 10 bits, histograms in shared memory, a block suffix scan to
// pick the digit) finds the k-th largest key T and how many tokens equal to T
// to take. One pass then takes every key > T (in any order: warp-aggregated
// atomics) and the first keys == T in token order (block prefix sums). A
// bitonic sort of the (key, token) pairs orders the result: strides of 64 and
// more through shared memory, strides of 32 and less in registers.
#include <cuda_runtime.h>

#include <cstdint>

#include "mqa_logits.h"
#include "ptx.cuh"

namespace mqa {

constexpr int kTopkThreads = 1024;
constexpr int kTopkBins = 2048;        // widest radix digit: 11 bits
constexpr int kTopkCacheKeys = 16384;  // keys cached in shared memory (64 KB)
constexpr int kTopkMinSort = 64;       // one warp's segment: 2 elements a lane

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

// Bitonic compare-exchange of this lane's element (global index i, value v)
// with the element i ^ stride held by lane ^ stride (stride < 32). The pair
// sorts descending when its lower index has bit `size` clear.
__device__ __forceinline__ uint64_t bitonic_lane_step(uint64_t v, int i, int stride, int size) {
    const uint64_t p = __shfl_xor_sync(0xffffffffu, v, stride);
    const bool lower = (i & stride) == 0;
    const bool desc = ((i & ~stride) & size) == 0;
    const uint64_t hi = v > p ? v : p, lo = v > p ? p : v;
    return (lower == desc) ? hi : lo;
}

// Strides 32, 16, ..., 1 of bitonic merge step `size` on one 64-element
// segment held as a (index base + lane) and b (base + 32 + lane).
__device__ __forceinline__ void bitonic_warp_merge(uint64_t& a, uint64_t& b, int base, int lane,
                                                   int size, int top_stride) {
    if (top_stride >= 32) {  // in-thread pair (base + lane, base + lane + 32)
        const bool desc = ((base + lane) & size) == 0;
        if (desc ? (a < b) : (a > b)) {
            const uint64_t t = a;
            a = b;
            b = t;
        }
    }
    for (int s = top_stride < 16 ? top_stride : 16; s > 0; s >>= 1) {
        a = bitonic_lane_step(a, base + lane, s, size);
        b = bitonic_lane_step(b, base + 32 + lane, s, size);
    }
}

__global__ void __launch_bounds__(kTopkThreads)
topk_kernel(const float* __restrict__ logits, const int32_t* __restrict__ context_lens,
            int next_n, int L, int k, int sort_n, int cache_n, int32_t* __restrict__ out) {
    extern __shared__ uint64_t sel[];  // [sort_n] (key << 32) | ~token, then keys[cache_n]
    uint32_t* keys = reinterpret_cast<uint32_t*>(sel + sort_n);
    __shared__ int hist[kTopkBins];
    __shared__ int ws[33];
    __shared__ int bcast[3];

    ptx::griddep_launch_dependents();
    ptx::griddep_wait();  // the logits may come from the previous kernel

    const int row = blockIdx.x;
    const int b = row / next_n, n = row - b * next_n;
    int c = __ldg(context_lens + b);
    c = c < 0 ? 0 : (c > L ? L : c);
    int cbn = c - next_n + 1 + n;
    cbn = cbn < 0 ? 0 : (cbn > c ? c : cbn);
    const float* x = logits + (int64_t)row * L;
    const int m = cbn < k ? cbn : k;  // tokens taken
    const int tid = threadIdx.x, nthr = blockDim.x, lane = tid & 31, warp = tid >> 5;
    const bool cached = cbn <= cache_n;

    if (cbn <= k) {
        // every valid token is taken
        for (int t = tid; t < cbn; t += nthr)
            sel[t] = ((uint64_t)topk_key(__ldg(x + t)) << 32) | (uint32_t)(~(uint32_t)t);
    } else {
        uint32_t prefix = 0, mask = 0;
        int remaining = k;  // still to take among keys matching `prefix`
#pragma unroll
        for (int p = 0; p < 3; ++p) {
            const int sh = p == 0 ? 21 : (p == 1 ? 10 : 0);  // digits: bits 31-21, 20-10, 9-0
            const int nb = p == 2 ? 1024 : 2048;
            for (int i = tid; i < nb; i += nthr) hist[i] = 0;
            __syncthreads();
            if (p == 0) {
                // first read of the row: four loads in flight a thread, keys
                // cached for the later passes
                for (int t0 = tid; t0 < cbn; t0 += 4 * nthr) {
                    float v[4];
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int t = t0 + j * nthr;
                        v[j] = t < cbn ? __ldg(x + t) : 0.f;
                    }
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int t = t0 + j * nthr;
                        if (t < cbn) {
                            const uint32_t key = topk_key(v[j]);
                            if (cached) keys[t] = key;
                            atomicAdd(&hist[key >> 21], 1);
                        }
                    }
                }
            } else {
                for (int t = tid; t < cbn; t += nthr) {
                    const uint32_t key = cached ? keys[t] : topk_key(__ldg(x + t));
                    if ((key & mask) == prefix) atomicAdd(&hist[(key >> sh) & (nb - 1)], 1);
                }
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
            if (tid == 0) bcast[2] = 0;  // counter of the take pass below
            __syncthreads();
            prefix |= (uint32_t)bcast[0] << sh;
            mask |= (uint32_t)(nb - 1) << sh;
            remaining = bcast[1];
            __syncthreads();
        }
        const uint32_t T = prefix;  // keys > T are all taken ...
        const int take_eq = remaining;  // ... and the first take_eq keys == T
        const int n_gt = k - take_eq;   // slots [0, n_gt) for keys > T

        int base_eq = 0;
        for (int start = 0; start < cbn; start += nthr) {
            const int t = start + tid;
            const uint32_t key = t < cbn ? (cached ? keys[t] : topk_key(__ldg(x + t))) : 0u;
            const uint64_t packed = ((uint64_t)key << 32) | (uint32_t)(~(uint32_t)t);
            const bool gt = t < cbn && key > T;
            const unsigned bal = __ballot_sync(0xffffffffu, gt);
            if (bal) {
                int pos0 = 0;
                if (lane == 0) pos0 = atomicAdd(&bcast[2], __popc(bal));
                pos0 = __shfl_sync(0xffffffffu, pos0, 0);
                if (gt) sel[pos0 + __popc(bal & ((1u << lane) - 1u))] = packed;
            }
            if (base_eq < take_eq) {  // uniform over the CTA
                const bool eq = t < cbn && key == T;
                if (__syncthreads_or(eq)) {
                    int neq;
                    const int rank = base_eq + block_exscan(eq ? 1 : 0, ws, neq);
                    if (eq && rank < take_eq) sel[n_gt + rank] = packed;
                    base_eq += neq;
                }
            }
        }
    }
    const int sort_len = sort_n;
    for (int i = m + tid; i < sort_len; i += nthr) sel[i] = 0ull;  // sorts last
    __syncthreads();

    // bitonic sort, descending (key descending, then token ascending). Warp w
    // owns 64-element segments w, w + 32, ...: lane l holds elements l and
    // l + 32 of the segment for the in-register strides.
    const int nseg = sort_len >> 6, nwarps = nthr >> 5;
    for (int seg = warp; seg < nseg; seg += nwarps) {
        const int base = seg << 6;
        uint64_t a = sel[base + lane], bv = sel[base + 32 + lane];
        for (int size = 2; size <= 64; size <<= 1) bitonic_warp_merge(a, bv, base, lane, size, size >> 1);
        sel[base + lane] = a;
        sel[base + 32 + lane] = bv;
    }
    __syncthreads();
    for (int size = 128; size <= sort_len; size <<= 1) {
        for (int stride = size >> 1; stride >= 64; stride >>= 1) {
            for (int i = tid; i < (sort_len >> 1); i += nthr) {
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
        for (int seg = warp; seg < nseg; seg += nwarps) {
            const int base = seg << 6;
            uint64_t a = sel[base + lane], bv = sel[base + 32 + lane];
            bitonic_warp_merge(a, bv, base, lane, size, 32);
            sel[base + lane] = a;
            sel[base + 32 + lane] = bv;
        }
        __syncthreads();
    }

    int32_t* o = out + (int64_t)row * k;
    for (int i = tid; i < k; i += nthr)
        o[i] = i < m ? (int32_t)(~(uint32_t)(sel[i] & 0xffffffffull)) : -1;
}

// Host launcher: one CTA per row; sort_n = next power of two >= k (at least
// one 64-element segment); keys of rows up to min(L, 16384) valid tokens are
// cached in shared memory. Launched with programmatic dependent launch, so
// it may start while the logits kernel before it drains.
int launch_topk(const float* logits, const int32_t* context_lens, int batch, int next_n, int L,
                int k, int32_t* out, void* stream) {
    int sort_n = kTopkMinSort;
    while (sort_n < k) sort_n <<= 1;
    const int cache_n = L < kTopkCacheKeys ? L : kTopkCacheKeys;
    const size_t smem = (size_t)sort_n * 8 + (size_t)cache_n * 4;
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, topk_kernel);
    if (e != cudaSuccess) return (int)e;
    if (fa.maxDynamicSharedSizeBytes < (int)smem) {
        e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smem);
        if (e != cudaSuccess) return (int)e;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(batch * next_n));
    cfg.blockDim = dim3(kTopkThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = static_cast<cudaStream_t>(stream);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return (int)cudaLaunchKernelEx(&cfg, topk_kernel, logits, context_lens, next_n, L, k, sort_n,
                                   cache_n, out);
}

}  // namespace mqa
