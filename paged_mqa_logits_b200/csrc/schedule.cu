// Split schedule for the persistent logits kernels, computed on the GPU.
//
// The page "[flashinfer] Blackwell 아키텍처를 위한 고성능 Paged MQA Logits 커널
// 도입", section 1 (the partition search became a binary search instead of a
// linear scan) and section 2 (the per-call work assignment is computed on the
// device, so there is no host round trip and the call can be captured in a
// CUDA graph). Units are 256 tokens of one row ("general lessons" 1).
//
// One CTA: every thread sums the units of a contiguous chunk of rows, a block
// scan turns the chunk sums into the exclusive prefix P[0..B] in shared
// memory, and every schedule entry is found by an upper-bound binary search
// over P (equal prefixes belong to rows without units, which the search steps
// over, so such rows are never named).
#include <cuda_runtime.h>

#include <cstdint>
#include "ptx.cuh"
#include "mqa_logits.h"

namespace mqa {

constexpr int kScheduleThreads = 1024;

__global__ void __launch_bounds__(kScheduleThreads, 1)
schedule_kernel(const int32_t* __restrict__ context_lens, int batch, int num_ctas,
                int32_t* __restrict__ schedule) {
    extern __shared__ int32_t prefix[];  // [batch + 1]
    __shared__ int32_t warp_sums[kScheduleThreads / 32];

    ptx::griddep_launch_dependents();
    // While the previous kernel finishes: bring context_lens into L2 (a hint;
    // L2 is the point of coherence, so a later write by that kernel still wins).
    for (int l = threadIdx.x; l * 32 < batch; l += blockDim.x) ptx::prefetch_l2(context_lens + l * 32);
    ptx::griddep_wait();  // context_lens may come from the previous kernel

    const int tid = threadIdx.x;
    const int nthr = blockDim.x;
    const int per = (batch + nthr - 1) / nthr;
    const int r0 = min(batch, tid * per);
    const int r1 = min(batch, r0 + per);

    int local = 0;
    for (int r = r0; r < r1; ++r) {
        const int c = max(__ldg(context_lens + r), 0);
        local += (c + MQA_SCHEDULE_UNIT - 1) / MQA_SCHEDULE_UNIT;
    }

    // block-wide exclusive scan of `local`
    const int lane = tid & 31, warp = tid >> 5;
    int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    if (lane == 31) warp_sums[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int nw = nthr >> 5;
        int w = lane < nw ? warp_sums[lane] : 0;
        int wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o) wi += v;
        }
        if (lane < nw) warp_sums[lane] = wi - w;  // exclusive warp offsets
    }
    __syncthreads();
    int run = warp_sums[warp] + incl - local;
    for (int r = r0; r < r1; ++r) {
        prefix[r] = run;
        const int c = max(__ldg(context_lens + r), 0);
        run += (c + MQA_SCHEDULE_UNIT - 1) / MQA_SCHEDULE_UNIT;
    }
    if (r1 == batch && r0 < r1) prefix[batch] = run;
    if (batch == 0 && tid == 0) prefix[0] = 0;
    __syncthreads();

    const int total = prefix[batch];
    const int q = total / num_ctas, rem = total % num_ctas;
    for (int i = tid; i <= num_ctas; i += nthr) {
        const int start = i * q + min(i, rem);
        int row = batch, off = 0;
        if (start < total) {
            // first index with prefix > start, over prefix[0..batch]
            int lo = 0, hi = batch + 1;
            while (lo < hi) {
                const int mid = (lo + hi) >> 1;
                if (prefix[mid] <= start) lo = mid + 1; else hi = mid;
            }
            row = lo - 1;
            off = start - prefix[row];
        }
        schedule[2 * i] = row;
        schedule[2 * i + 1] = off;
    }
}

// Host launcher: one CTA, shared prefix of batch + 1 entries.
int launch_schedule(const int32_t* context_lens, int batch, int num_ctas, int32_t* schedule,
                    void* stream) {
    const uint32_t smem = (uint32_t)(batch + 1) * 4;
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, schedule_kernel);
    if (e != cudaSuccess) return (int)e;
    if (fa.maxDynamicSharedSizeBytes < (int)smem) {
        e = cudaFuncSetAttribute(schedule_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smem);
        if (e != cudaSuccess) return (int)e;
    }
    // Same shared-memory carveout as the logits kernels that follow, so the SMs
    // need no L1/shared reconfiguration between the two launches.
    if (fa.preferredShmemCarveout != 100) {
        e = cudaFuncSetAttribute(schedule_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 100);
        if (e != cudaSuccess) return (int)e;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(1);
    cfg.blockDim = dim3(batch > 256 ? kScheduleThreads : 256);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = static_cast<cudaStream_t>(stream);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return (int)cudaLaunchKernelEx(&cfg, schedule_kernel, context_lens, batch, num_ctas, schedule);
}

}  // namespace mqa
