// Block-scaled FP4 paged MQA logits on sm_100a (the page "[flashinfer]
// Blackwell 아키텍처를 위한 고성능 Paged MQA Logits 커널 도입": introduction,
// fp4_paged_mqa_logits, run here as a true FP4 MMA).
//
// Both operands are NVFP4: e2m1 codes (two per byte, even element in the low
// nibble) with one unsigned e4m3 scale per 16 consecutive elements. K comes
// from the FP4 page format (codes, then scales); q comes per (b, n) row in the
// same shape ([H][D/2] codes, then [H][D/16] scales). The tensor core applies
// both sets of scales inside the dot product (tcgen05.mma kind::mxf4nvf4,
// scale_vec::4X), so nothing is dequantised: D/64 instructions per 128-token
// tile, accumulating in fp32 in TMEM. There is no per-token scale (s_t = 1).
//
// The skeleton is the FP8 kernel's (persistent, one CTA per SM, the shared
// work table, three producer warps, three epilogue groups, the tail warp and
// the builder warp); what differs is the MMA warp. The block-scaled MMA reads
// its scales from TMEM in a fixed arrangement: for a 128-row operand and one
// instruction (64 elements of K), row m's four one-byte scales sit in lane
// m % 32 (of every lane quarter), column m / 32. The scales arrive from HBM
// token-major ([rows][D/16] bytes), so the whole MMA warp first rearranges
// them in shared memory into 512-byte blocks (byte (m % 32) * 16 + (m / 32) * 4
// + j holds scale j of row m) and lane 0 copies each block to TMEM with
// tcgen05.cp.32x128b.warpx4, then issues the MMAs (a tcgen05.cp and the
// tcgen05.mma that reads it are executed in issue order).
//
// TMEM: nacc accumulator slots, then the K scale blocks of each ring stage
// (2 tiles x D/64 blocks x 4 columns; a stage's blocks are rewritten only
// after the stage was refilled, i.e. after its previous MMAs completed), then
// the q scale blocks of the two q buffers (rewritten only after the row two
// rows back was released, which needs its MMAs to have completed).
#include <cuda_runtime.h>

#include <cstdint>
#include "common.cuh"
#include "epilogue.cuh"

namespace mqa {

constexpr int kEpiGroupsN = 3;
constexpr int kMmaWarpN = kProducers;                         // 3
constexpr int kEpiWarpN = kProducers + 1;                     // 4..15
constexpr int kTailWarpN = kEpiWarpN + 4 * kEpiGroupsN;       // 16
constexpr int kBuildWarpN = kTailWarpN + 1;                   // 17
constexpr int kNvfp4Threads = 32 * (kBuildWarpN + 1);
static_assert(kProducers + 1 + 4 * kEpiGroupsN == kTableUsers, "table users");

// TMEM columns of the scale blocks that follow the accumulators.
__host__ __device__ inline int nvfp4_sf_cols(int D, int stages) {
    return (stages * 2 + 2) * (D / 64) * 4;
}

// Accumulator slots that fit in 512 columns next to the scale blocks (a power
// of two, so a tile's slot and use are a mask and a shift).
__host__ __device__ inline int nvfp4_acc_slots(int D, int npad, int stages) {
    const int n = (512 - nvfp4_sf_cols(D, stages)) / acc_stride(npad);
    int p = 1;
    while (p * 2 <= n && p * 2 <= kMaxAccSlots) p *= 2;
    return p;
}

// Shared-memory matrix descriptor of one 512-byte scale block: 32 rows of 16
// bytes, no swizzle (8-row core matrices 128 bytes apart).
__device__ __forceinline__ uint64_t sf_block_desc(const void* p) {
    return ptx::smem_desc(ptx::smem_u32(p), 128, 128, ptx::SW_NONE);
}

template <int H, int D>
__global__ void __launch_bounds__(kNvfp4Threads, 1)
nvfp4_logits_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_q,
                    const KernelArgs a) {
    constexpr int kRowBytes = D / 2;                 // packed codes per token / q row
    constexpr int kScaleBytes = D / 16;              // scales per token / q row
    constexpr int kScaleWords = kScaleBytes / 4;     // = D / 64 = K steps per tile
    constexpr int kKSteps = D / 64;                  // MMA K = 64 e2m1 per instruction
    constexpr int kStageBytes = kUnit * kRowBytes;
    constexpr int kTileBytes = kTile * kRowBytes;
    constexpr uint32_t kSwz = kRowBytes == 64 ? ptx::SW_64B : ptx::SW_32B;
    constexpr uint32_t kSBO = 8 * kRowBytes;         // bytes between 8-row core-matrix groups
    static_assert(kScaleWords == kKSteps, "one 4-byte scale word per K step");

    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int NS = a.num_stages;
    const int npad = a.npad;
    const int astride = acc_stride(npad);
    const int nacc = nvfp4_acc_slots(D, npad, NS);
    const int acc_shift = 31 - __clz(nacc);
    const Nvfp4Smem L = nvfp4_smem_layout(D, npad, NS);
    uint8_t* kst = base + L.kst;
    uint8_t* qbuf = base + L.qbuf;
    uint8_t* ksf = base + L.ksf;
    uint8_t* qsf = base + L.qsf;
    const uint32_t* kraw = reinterpret_cast<const uint32_t*>(base + L.kraw);
    const uint32_t* qraw = reinterpret_cast<const uint32_t*>(base + L.qraw);
    float* wbuf = reinterpret_cast<float*>(base + L.wbuf);
    uint64_t* full = reinterpret_cast<uint64_t*>(base + L.bars);
    uint64_t* empty = full + NS;
    uint64_t* qfull = empty + NS;
    uint64_t* qempty = qfull + 2;
    uint64_t* drain = qempty + 2;
    uint64_t* tbars = drain + 1;                 // table full[2], empty[2]
    uint64_t* accfull = tbars + 4;
    uint64_t* accempty = accfull + kMaxAccSlots;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(base + L.misc);
    volatile CtaFlags* cf = reinterpret_cast<volatile CtaFlags*>(base + L.misc + 8);
    const Table T = table_view(base + L.table, tbars, a);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int cta = blockIdx.x;
    const uint32_t ksf_col0 = (uint32_t)(nacc * astride);
    const uint32_t qsf_col0 = ksf_col0 + (uint32_t)(NS * 2 * kKSteps * 4);
    uint32_t ncols = 32;
    while (ncols < qsf_col0 + 2u * kKSteps * 4) ncols <<= 1;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            ptx::mbar_init(&full[s], 1);
            ptx::mbar_init(&empty[s], 1);  // released by the MMA's commit
        }
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(&qfull[i], 1);
            ptx::mbar_init(&qempty[i], 1 + 4 * kEpiGroupsN);
            ptx::mbar_init(&T.full[i], 32);
            ptx::mbar_init(&T.empty[i], kTableUsers);
        }
        for (int i = 0; i < kMaxAccSlots; ++i) {
            ptx::mbar_init(&accfull[i], 1);
            ptx::mbar_init(&accempty[i], 4);
        }
        ptx::mbar_init(drain, 1);
        cf->abort = 0;
        cf->consumed = 0;
        cf->q_seen = 0;
        ptx::fence_mbar_init();
        ptx::prefetch_tmap(&tm_k);
        ptx::prefetch_tmap(&tm_q);
    }
    __syncwarp();
    if (warp == kMmaWarpN) {
        ptx::tmem_alloc(tmem_holder, ncols);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    ptx::griddep_launch_dependents();
    if (warp >= kEpiWarpN && warp <= kTailWarpN)  // idle at first: warm L2 with the small inputs
        warm_inputs(a, cta, threadIdx.x - 32 * kEpiWarpN, 32 * (kTailWarpN + 1 - kEpiWarpN));
    ptx::griddep_wait();  // inputs (schedule, context_lens, ...) may come from the previous kernel

    // q codes of row b (all drafts, N = next_n * H rows) + their scales +
    // weights into q buffer q; codes + scales of page p of unit u into stage s
    const uint32_t q_row_bytes = (uint32_t)(a.heads * (kRowBytes + kScaleBytes));
    auto q_load = [&](int q, int b) {
        ptx::tma_load_3d(qbuf + q * npad * kRowBytes, &tm_q, &qfull[q], 0, 0, b * a.next_n);
        for (int n = 0; n < a.next_n; ++n)
            ptx::bulk_load(base + L.qraw + q * 128 * kScaleBytes + n * a.heads * kScaleBytes,
                           a.q + (int64_t)(b * a.next_n + n) * q_row_bytes + a.heads * kRowBytes,
                           (uint32_t)(a.heads * kScaleBytes), &qfull[q]);
        ptx::bulk_load(wbuf + q * 256, a.weights + (int64_t)b * a.hn, (uint32_t)(a.hn * 4),
                       &qfull[q]);
    };
    auto page_load = [&](int s, int u, int p, int rows, int row_off, int pg) {
        (void)u;
        ptx::tma_load_3d(kst + s * kStageBytes + p * rows * kRowBytes, &tm_k, &full[s], 0, row_off,
                         pg);
        ptx::bulk_load(base + L.kraw + (s * kUnit + p * rows) * kScaleBytes,
                       a.kv + (int64_t)pg * a.page_bytes + a.page_size * kRowBytes +
                           row_off * kScaleBytes,
                       (uint32_t)(rows * kScaleBytes), &full[s]);
    };
    const uint32_t row_bytes = (uint32_t)(kRowBytes + kScaleBytes);
    const uint32_t q_bytes = (uint32_t)(a.hn * (kRowBytes + kScaleBytes) + a.hn * 4);
    const int first = builder_units(a, T, a.num_stages);

    if (warp < kProducers) {
        // ------------------------------------------------------------ producers
        producer_warp<kProducers>(a, T, warp, lane, first, full, empty, qfull, qempty, cf, row_bytes, q_bytes,
                      q_load, page_load);
    } else if (warp == kMmaWarpN) {
        // ------------------------------------------------------------ scales + MMA issuer
        const uint32_t idesc = ptx::instr_desc_mxf4nvf4(kTile, (uint32_t)npad);
        TableCursor cur;
        int qi = -1, s = 0, u = 0;
        uint32_t ph = 0;
        bool stop = false;
#ifdef MQA_DEBUG
        DebugWalk dw;
        debug_walk_begin(a, cta, dw);
#endif
        while (!stop && cur.next<true>(T, cf, a, lane) == 0) {
            const UnitDesc d = cur.desc(T);
            const int info = cur.info(T);
#ifdef MQA_DEBUG
            if (lane == 0) debug_check_unit(a, d, info, dw);
#endif
            if (info & 1) {  // a new row: release the previous q, wait for this one
                if (qi >= 0 && lane == 0) ptx::tc_commit(&qempty[qi & 1]);
                qi = info >> 1;
                const int q = qi & 1;
                if (!warp_wait(&qfull[q], (uint32_t)(qi >> 1) & 1, cf, a, lane)) break;
                if (lane == 0) cf->q_seen = qi + 1;
                // q scales [N rows][D/16] -> one 512-byte block per K step
                uint32_t* dst = reinterpret_cast<uint32_t*>(qsf + q * kKSteps * 512);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int m = lane + 32 * j;
#pragma unroll
                    for (int i = 0; i < kKSteps; ++i)
                        dst[i * 128 + lane * 4 + j] =
                            m < a.hn ? qraw[q * 128 * kScaleWords + m * kScaleWords + i] : 0u;
                }
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                __syncwarp();
                if (lane == 0) {
                    ptx::tc_fence_after();
#pragma unroll
                    for (int i = 0; i < kKSteps; ++i)
                        ptx::tmem_cp_32x128b_x4(tmem + qsf_col0 + (uint32_t)((q * kKSteps + i) * 4),
                                                sf_block_desc(qsf + (q * kKSteps + i) * 512));
                }
            }
            if (!warp_wait(&full[s], ph, cf, a, lane)) break;
            if (lane == 0) cf->consumed = u + 1;
            const int nt = unit_tiles(d);
            // the unit's K scales [256 tokens][D/16] -> per tile, one block per K step
            // (lane l gathers tokens l, l + 32, l + 64, l + 96 of a tile: one
            // load of all of a token's scale words each, then one 16-byte store
            // per block)
            {
                uint4* dst = reinterpret_cast<uint4*>(ksf + s * 2 * kKSteps * 512);
                const uint32_t* src = kraw + s * kUnit * kScaleWords;
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    if (k < nt) {
                        uint32_t w[4][kScaleWords];
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const uint32_t* tok = src + (k * kTile + lane + 32 * j) * kScaleWords;
                            if constexpr (kScaleWords == 2) {
                                const uint2 v = *reinterpret_cast<const uint2*>(tok);
                                w[j][0] = v.x;
                                w[j][kScaleWords - 1] = v.y;
                            } else {
                                w[j][0] = tok[0];
                            }
                        }
#pragma unroll
                        for (int i = 0; i < kKSteps; ++i)
                            dst[(k * kKSteps + i) * 32 + lane] = make_uint4(w[0][i], w[1][i], w[2][i], w[3][i]);
                    }
                }
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
            int ok = 1;
            if (lane == 0) {
                ptx::tc_fence_after();
                for (int k = 0; k < nt; ++k)
#pragma unroll
                    for (int i = 0; i < kKSteps; ++i)
                        ptx::tmem_cp_32x128b_x4(
                            tmem + ksf_col0 + (uint32_t)(((s * 2 + k) * kKSteps + i) * 4),
                            sf_block_desc(ksf + ((s * 2 + k) * kKSteps + i) * 512));
                const uint32_t qsf_t = tmem + qsf_col0 + (uint32_t)((qi & 1) * kKSteps * 4);
                const uint32_t b_base = ptx::smem_u32(qbuf + (qi & 1) * npad * kRowBytes);
                for (int k = 0; k < nt; ++k) {
                    const int tile = d.tile + k;
                    const int slot = tile & (nacc - 1);
                    const uint32_t use = (uint32_t)(tile >> acc_shift);
                    if (!wait_bounded(&accempty[slot], (use & 1) ^ 1, cf, a)) { ok = 0; break; }
                    ptx::tc_fence_after();
                    const uint32_t d_tmem = tmem + (uint32_t)(slot * astride);
                    const uint32_t a_base = ptx::smem_u32(kst + s * kStageBytes + k * kTileBytes);
#pragma unroll
                    for (int i = 0; i < kKSteps; ++i)  // K advances by 32 bytes per step
                        ptx::mma_mxf4nvf4_ss(
                            d_tmem, ptx::smem_desc(a_base + 32 * i, 0, kSBO, kSwz),
                            ptx::smem_desc(b_base + 32 * i, 0, kSBO, kSwz), idesc,
                            tmem + ksf_col0 + (uint32_t)(((s * 2 + k) * kKSteps + i) * 4),
                            qsf_t + (uint32_t)(i * 4), i > 0 ? 1u : 0u);
                    ptx::tc_commit(&accfull[slot]);
                }
                if (ok) ptx::tc_commit(&empty[s]);  // the stage is free once these MMAs complete
            }
            stop = __shfl_sync(0xffffffffu, ok, 0) == 0;
            if (++s == NS) { s = 0; ph ^= 1; }
            ++u;
        }
        if (lane == 0) {
            // all MMAs and copies issued by this thread are complete before TMEM is freed
            ptx::tc_commit(drain);
            wait_drain(drain, 0, a);
        }
        __syncwarp();  // reconverge before the CTA barrier (an aligned barrier)
    } else if (warp < kTailWarpN) {
        // ------------------------------------------------------------ epilogue
        const int group = (warp - kEpiWarpN) >> 2;  // takes tiles i with i % kEpiGroupsN == group
        const int quarter = warp & 3;       // TMEM lane quarter this warp may access
        const int r = quarter * 32 + lane;  // token within the tile
        const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
        TableCursor cur;
        int qi = -1;
        bool stop = false;
        while (!stop && cur.next<true>(T, cf, a, lane) == 0) {
            const UnitDesc d = cur.desc(T);
            const int info = cur.info(T);
            if (info & 1) {
                if (qi >= 0) {
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(&qempty[qi & 1]);
                }
                qi = info >> 1;
                if (!warp_wait(&qfull[qi & 1], (uint32_t)(qi >> 1) & 1, cf, a, lane)) break;
            }
            const int nt = unit_tiles(d);
            for (int k = 0; k < nt; ++k) {
                const int tile = d.tile + k;
                if (tile % kEpiGroupsN != group) continue;
                const int slot = tile & (nacc - 1);
                if (!warp_wait(&accfull[slot], (uint32_t)(tile >> acc_shift) & 1, cf, a, lane)) {
                    stop = true;
                    break;
                }
                ptx::tc_fence_after();
                const int t = d.t0 + k * kTile + r;
                float* orow = a.out + ((int64_t)d.b * a.next_n) * a.out_len + t;
                epilogue_tile<H>(lane_base + (uint32_t)(slot * astride), wbuf + (qi & 1) * 256,
                                 1.0f, a.next_n, d.ctx, t, a.out_len, orow, &accempty[slot], lane);
            }
        }
    } else if (warp == kTailWarpN) {
        // ------------------------------------------------------------ tail fill
        if (a.flags & MQA_FLAG_VALIDATE) check_schedule(a, cta, lane);
        tail_fill(a, cta, 0, 1, lane);
    } else {
        // ------------------------------------------------------------ work table
        build_table(a, cta, T, cf, lane, first, full, qfull, row_bytes, q_bytes, q_load, page_load);
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarpN) {
        __syncwarp();
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, ncols);
    }
}

// ---------------------------------------------------------------- host launcher
template <typename Kernel>
static int launch_instance(Kernel kernel, int threads, const LaunchSpec& ls,
                           const CUtensorMap& tm_k, const CUtensorMap& tm_q,
                           const KernelArgs& args) {
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, kernel);
    if (e != cudaSuccess) return (int)e;
    if (fa.maxDynamicSharedSizeBytes < (int)ls.smem) {
        e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ls.smem);
        if (e != cudaSuccess) return (int)e;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(ls.grid);
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = ls.smem;
    cfg.stream = static_cast<cudaStream_t>(ls.stream);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = ls.pdl ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return (int)cudaLaunchKernelEx(&cfg, kernel, tm_k, tm_q, args);
}

int launch_nvfp4_logits(int H, int D, const LaunchSpec& ls, const CUtensorMap& tm_k,
                        const CUtensorMap& tm_q, const KernelArgs& args) {
#define MQA_NVFP4_CASE(HH, DD)                                                               \
    case HH * 1000 + DD:                                                                     \
        return launch_instance(&nvfp4_logits_kernel<HH, DD>, kNvfp4Threads, ls, tm_k, tm_q,  \
                               args);
    switch (H * 1000 + D) {
        MQA_NVFP4_CASE(4, 64) MQA_NVFP4_CASE(4, 128)
        MQA_NVFP4_CASE(8, 64) MQA_NVFP4_CASE(8, 128)
        MQA_NVFP4_CASE(16, 64) MQA_NVFP4_CASE(16, 128)
        MQA_NVFP4_CASE(32, 64) MQA_NVFP4_CASE(32, 128)
        MQA_NVFP4_CASE(64, 64) MQA_NVFP4_CASE(64, 128)
        MQA_NVFP4_CASE(128, 64) MQA_NVFP4_CASE(128, 128)
    }
#undef MQA_NVFP4_CASE
    return (int)cudaErrorInvalidValue;
}

}  // namespace mqa
