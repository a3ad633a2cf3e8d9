// Gather-only diagnostic of the FP8 path: the FP8 kernel's work table,
// builder and producer (common.cuh) move exactly the K rows and q tiles the
// logits kernel moves, with the same ring of shared-memory stages and the
// same tensor maps, but nothing computes: a consumer warp releases each stage
// as soon as it lands. Timing it on a workload gives the copy-only time of
// that workload's page gather, the floor the logits kernel's data path can
// reach with this issue scheme. Nothing is written to `out`.
//
// Three warps: producer (warp 0), consumer (warp 1: walks the table, takes
// each row's q buffer and each stage, releases them), builder (warp 2). Every
// wait is bounded, as in the logits kernels.
#include <cuda_runtime.h>

#include <cstdint>
#include "common.cuh"

namespace mqa {

constexpr int kGatherThreads = 96;
constexpr int kGatherTableUsers = 2;  // producer, consumer

template <int D>
__global__ void __launch_bounds__(kGatherThreads, 1)
fp8_gather_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_q,
                  const KernelArgs a) {
    constexpr int kStageBytes = kUnit * D;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int NS = a.num_stages;
    const int npad = a.npad;
    const Fp8Smem L = fp8_smem_layout(D, npad, NS);
    uint8_t* kst = base + L.kst;
    uint8_t* qbuf = base + L.qbuf;
    float* wbuf = reinterpret_cast<float*>(base + L.wbuf);
    uint64_t* full = reinterpret_cast<uint64_t*>(base + L.bars);
    uint64_t* empty = full + NS;
    uint64_t* qfull = empty + NS;
    uint64_t* qempty = qfull + 2;
    uint64_t* tbars = qempty + 2;  // table full[2], empty[2]
    volatile CtaFlags* cf = reinterpret_cast<volatile CtaFlags*>(base + L.misc + 8);
    const Table T = table_view(base + L.table, tbars, a);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int cta = blockIdx.x;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            ptx::mbar_init(&full[s], 1);
            ptx::mbar_init(&empty[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(&qfull[i], 1);
            ptx::mbar_init(&qempty[i], 1);
            ptx::mbar_init(&T.full[i], 32);
            ptx::mbar_init(&T.empty[i], kGatherTableUsers);
        }
        cf->abort = 0;
        cf->consumed = 0;
        cf->q_seen = 0;
        ptx::fence_mbar_init();
        ptx::prefetch_tmap(&tm_k);
        ptx::prefetch_tmap(&tm_q);
    }
    __syncthreads();
    ptx::griddep_launch_dependents();
    ptx::griddep_wait();

    auto q_load = [&](int q, int b) {
        ptx::tma_load_2d(qbuf + q * npad * D, &tm_q, &qfull[q], 0, b * a.hn);
        ptx::bulk_load(wbuf + q * 256, a.weights + (int64_t)b * a.hn, (uint32_t)(a.hn * 4),
                       &qfull[q]);
    };
    auto page_load = [&](int s, int u, int p, int rows, int row_off, int pg) {
        (void)u;
        ptx::tma_load_3d(kst + s * kStageBytes + p * rows * D, &tm_k, &full[s], 0, row_off, pg);
    };
    const uint32_t row_bytes = (uint32_t)D;
    const uint32_t q_bytes = (uint32_t)(npad * D + a.hn * 4);
    const int first = builder_units(a, T, 1);

    if (warp == 0) {
        producer_warp<1>(a, T, 0, lane, first, full, empty, qfull, qempty, cf, row_bytes, q_bytes,
                         q_load, page_load);
    } else if (warp == 1) {
        TableCursor cur;
        int qi = -1, s = 0, u = 0;
        uint32_t ph = 0;
        while (cur.next<true>(T, cf, a, lane) == 0) {
            const int info = cur.info(T);
            if (info & 1) {  // a new row: release the previous q, wait for this one
                if (qi >= 0 && lane == 0) ptx::mbar_arrive(&qempty[qi & 1]);
                qi = info >> 1;
                if (!warp_wait(&qfull[qi & 1], (uint32_t)(qi >> 1) & 1, cf, a, lane)) break;
                if (lane == 0) cf->q_seen = qi + 1;
            }
            if (!warp_wait(&full[s], ph, cf, a, lane)) break;
            if (lane == 0) {
                cf->consumed = u + 1;
                ptx::mbar_arrive(&empty[s]);
            }
            __syncwarp();
            if (++s == NS) { s = 0; ph ^= 1; }
            ++u;
        }
    } else {
        build_table(a, cta, T, cf, lane, first, full, qfull, row_bytes, q_bytes, q_load, page_load);
    }
    __syncthreads();
}

int launch_fp8_gather(int D, const LaunchSpec& ls, const CUtensorMap& tm_k, const CUtensorMap& tm_q,
                      const KernelArgs& args) {
    auto go = [&](auto kernel) -> int {
        cudaFuncAttributes fa;
        cudaError_t e = cudaFuncGetAttributes(&fa, kernel);
        if (e != cudaSuccess) return (int)e;
        if (fa.maxDynamicSharedSizeBytes < (int)ls.smem) {
            e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)ls.smem);
            if (e != cudaSuccess) return (int)e;
        }
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(ls.grid);
        cfg.blockDim = dim3(kGatherThreads);
        cfg.dynamicSmemBytes = ls.smem;
        cfg.stream = static_cast<cudaStream_t>(ls.stream);
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = ls.pdl ? 1 : 0;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        return (int)cudaLaunchKernelEx(&cfg, kernel, tm_k, tm_q, args);
    };
    switch (D) {
        case 32: return go(fp8_gather_kernel<32>);
        case 64: return go(fp8_gather_kernel<64>);
        case 128: return go(fp8_gather_kernel<128>);
    }
    return (int)cudaErrorInvalidValue;
}

}  // namespace mqa
