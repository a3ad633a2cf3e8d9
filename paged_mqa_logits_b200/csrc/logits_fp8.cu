// FP8 paged MQA logits on sm_100a (the page "[flashinfer] Blackwell 아키텍처를
// 위한 고성능 Paged MQA Logits 커널 도입": introduction, fp8_paged_mqa_logits;
// section 1: persistent TMA + UMMA kernel, zero-length rows skipped in the task
// iterator, epilogue caching sized by register footprint).
//
// One persistent CTA per SM; one pipeline stage is one 256-token schedule unit
// (two 128-token MMA tiles). 16 warps:
//   warps 0-11  epilogue, three groups of four warps taking tiles in turn
//               (tile i goes to group i mod 3): thread = token (its TMEM
//               lane); logit[n] = sum_h w[n,h] * max(s_t * acc[t, nH+h], 0),
//               -inf past the draft context (a select), one coalesced fp32
//               store per draft row. Each thread reads its token's fp32 scale
//               s_t straight from the page as soon as the group reaches the
//               unit, well before the tile's accumulator is ready.
//   warp 12     the producer: every unit of the work table in unit order (so
//               the oldest unit's loads are always ahead in the memory
//               queues): the K rows of the unit's pages (3-D tensor map,
//               swizzled for the MMA) into a ring stage, plus an L2 prefetch
//               of the pages' scales for the epilogue; it also loads each
//               row's q tile and weights (from the third row on).
//   warp 13     MMA issuer (and TMEM owner): per tile, acc[t, c] =
//               sum_d k[t,d] q[c,d] with c = n*H + h, as D/32 tcgen05
//               kind::f8f6f4 instructions (M = 128 tokens, N = H*next_n
//               padded to 16, fp32 in a ring of TMEM accumulator slots); it
//               frees each K stage once its MMAs complete.
//   warp 14     the -inf tail of every output row past its last tile.
//   warp 15     builds the work table (build_table) and issues the loads of
//               the first unit and of the first two rows' q.
// Before the grid-dependency wait, the epilogue and tail warps warm L2 with
// the small inputs (warm_inputs).
// Every wait is bounded (MQA_STATUS_TIMEOUT, never a trap).
#include <cuda_runtime.h>

#include <cstdint>
#include "common.cuh"
#include "epilogue.cuh"

namespace mqa {

constexpr int kEpiGroups = 3;
constexpr int kProdWarp = 4 * kEpiGroups;                   // 12
constexpr int kMmaWarp = kProdWarp + 1;                     // 13
constexpr int kTailWarp = kMmaWarp + 1;                     // 14
constexpr int kBuildWarp = kTailWarp + 1;                   // 15
constexpr int kFp8Threads = 32 * (kBuildWarp + 1);
constexpr int kFp8TableUsers = 4 * kEpiGroups + 2;          // epilogue, producer, MMA

// 32-bit float global load cached in L2 only.
__device__ __forceinline__ float ld_cg_f32(const void* p) {
    float v;
    asm volatile("ld.global.cg.f32 %0, [%1];" : "=f"(v) : "l"(reinterpret_cast<uint64_t>(p)));
    return v;
}

template <int H, int D>
__global__ void __launch_bounds__(kFp8Threads, 1)
fp8_logits_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_q,
                  const KernelArgs a) {
    constexpr uint32_t kSwz = D == 128 ? ptx::SW_128B : (D == 64 ? ptx::SW_64B : ptx::SW_32B);
    constexpr uint32_t kSBO = 8 * D;          // bytes between 8-row core-matrix groups
    constexpr int kStageBytes = kUnit * D;
    constexpr int kTileBytes = kTile * D;
    constexpr int kKSteps = D / 32;           // MMA K = 32 e4m3 per instruction

    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int NS = a.num_stages;
    const int npad = a.npad;
    const int astride = acc_stride(npad);
    // TMEM accumulator slots: the largest power of two <= min(8, 512 / astride),
    // so a tile's slot and use are a mask and a shift
    const int acc_shift = 31 - __clz(min(kMaxAccSlots, 512 / astride));
    const int nacc = 1 << acc_shift;
    const Fp8Smem L = fp8_smem_layout(D, npad, NS);
    uint8_t* kst = base + L.kst;
    uint8_t* qbuf = base + L.qbuf;
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
    uint32_t ncols = 32;
    while (ncols < (uint32_t)(nacc * astride)) ncols <<= 1;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            ptx::mbar_init(&full[s], 1);
            ptx::mbar_init(&empty[s], 1);  // released by the MMA's commit
        }
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(&qfull[i], 1);
            ptx::mbar_init(&qempty[i], 1 + 4 * kEpiGroups);
            ptx::mbar_init(&T.full[i], 32);
            ptx::mbar_init(&T.empty[i], kFp8TableUsers);
        }
        for (int i = 0; i < kMaxAccSlots; ++i) {
            ptx::mbar_init(&accfull[i], 1);
            ptx::mbar_init(&accempty[i], 4);
        }
        ptx::mbar_init(drain, 1);
        cf->abort = 0;
        cf->consumed = 0;
        cf->q_seen = 0;
#ifdef MQA_DEBUG
        for (int i = 0; i < kDbgSlots; ++i) g_mqa_dbg[i] = -1;
#endif
        ptx::fence_mbar_init();
        ptx::prefetch_tmap(&tm_k);
        ptx::prefetch_tmap(&tm_q);
    }
    __syncwarp();
    if (warp == kMmaWarp) {
        ptx::tmem_alloc(tmem_holder, ncols);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    ptx::griddep_launch_dependents();
    if (warp < kProdWarp || warp == kTailWarp)  // idle at first: warm L2 with the small inputs
        warm_inputs(a, cta, warp == kTailWarp ? 32 * kProdWarp + lane : (int)threadIdx.x,
                    32 * (kProdWarp + 1));
    ptx::griddep_wait();  // inputs (schedule, context_lens, ...) may come from the previous kernel

    // q tile + weights of row b into q buffer q; K rows of page p of unit u
    // into stage s, and an L2 prefetch of the same rows' fp32 scales (read by
    // the epilogue, not by the TMA)
    auto q_load = [&](int q, int b) {
        ptx::tma_load_2d(qbuf + q * npad * D, &tm_q, &qfull[q], 0, b * a.hn);
        ptx::bulk_load(wbuf + q * 256, a.weights + (int64_t)b * a.hn, (uint32_t)(a.hn * 4),
                       &qfull[q]);
    };
    auto page_load = [&](int s, int u, int p, int rows, int row_off, int pg) {
        (void)u;
        ptx::tma_load_3d(kst + s * kStageBytes + p * rows * D, &tm_k, &full[s], 0, row_off, pg);
        const uint8_t* sc = a.kv + (int64_t)pg * a.page_bytes + (int64_t)a.page_size * D + row_off * 4;
        for (int l = 0; l < rows * 4; l += 128) ptx::prefetch_l2(sc + l);
    };
    const uint32_t row_bytes = (uint32_t)D;
    const uint32_t q_bytes = (uint32_t)(npad * D + a.hn * 4);
    const int first = builder_units(a, T, 1);
    const int sh = a.ps_shift;

    if (warp == kProdWarp) {
        // ------------------------------------------------------------ producer
        producer_warp<1>(a, T, 0, lane, first, full, empty, qfull, qempty, cf, row_bytes, q_bytes,
                         q_load, page_load);
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc = ptx::instr_desc(0, 0, kTile, (uint32_t)npad);
            TableCursor cur;
            int qi = -1, s = 0, u = 0;
            uint32_t ph = 0;
#ifdef MQA_DEBUG
            DebugWalk dw;
            debug_walk_begin(a, cta, dw);
#endif
            while (cur.next<false>(T, cf, a, 0) == 0) {
                const UnitDesc d = cur.desc(T);
                const int info = cur.info(T);
#ifdef MQA_DEBUG
                debug_check_unit(a, d, info, dw);
#endif
                if (info & 1) {  // a new row: release the previous q, wait for this one
                    if (qi >= 0) ptx::tc_commit(&qempty[qi & 1]);
                    qi = info >> 1;
                    if (!wait_bounded(&qfull[qi & 1], (uint32_t)(qi >> 1) & 1, cf, a)) break;
                    cf->q_seen = qi + 1;
                }
                if (!wait_bounded(&full[s], ph, cf, a)) break;
                cf->consumed = u + 1;
                const uint64_t db =
                    ptx::smem_desc(ptx::smem_u32(qbuf + (qi & 1) * npad * D), 0, kSBO, kSwz);
                const int nt = unit_tiles(d);
                // both accumulator slots first, then the unit's MMAs back to back
                // (an MMA issues in ~60 cycles; waits between them cost as much)
                const int tile0 = d.tile;
                const int slot0 = tile0 & (nacc - 1), slot1 = (tile0 + 1) & (nacc - 1);
                if (!wait_bounded(&accempty[slot0], ((uint32_t)(tile0 >> acc_shift) & 1) ^ 1, cf, a))
                    break;
                if (nt > 1 &&
                    !wait_bounded(&accempty[slot1], ((uint32_t)((tile0 + 1) >> acc_shift) & 1) ^ 1, cf, a))
                    break;
                ptx::tc_fence_after();
                // K advances by 32 bytes per step: 2 in the descriptor's address field
                const uint64_t da0 = ptx::smem_desc(ptx::smem_u32(kst + s * kStageBytes), 0, kSBO, kSwz);
#pragma unroll
                for (int kk = 0; kk < kKSteps; ++kk)
                    ptx::mma_f8f6f4_ss(tmem + (uint32_t)(slot0 * astride), da0 + 2 * kk, db + 2 * kk,
                                       idesc, kk > 0 ? 1u : 0u);
                ptx::tc_commit(&accfull[slot0]);
                if (nt > 1) {
                    const uint64_t da1 = da0 + (kTileBytes >> 4);  // the second tile's rows
#pragma unroll
                    for (int kk = 0; kk < kKSteps; ++kk)
                        ptx::mma_f8f6f4_ss(tmem + (uint32_t)(slot1 * astride), da1 + 2 * kk,
                                           db + 2 * kk, idesc, kk > 0 ? 1u : 0u);
                    ptx::tc_commit(&accfull[slot1]);
                }
                ptx::tc_commit(&empty[s]);  // the stage is free once these MMAs complete
                if (++s == NS) { s = 0; ph ^= 1; }
                ++u;
            }
            // all MMAs issued by this thread are complete before TMEM is freed
            ptx::tc_commit(drain);
            wait_drain(drain, 0, a);
#ifdef MQA_DEBUG
            if (!cf->abort) {
                g_mqa_dbg[kDbgUnits] = dw.units;
                g_mqa_dbg[kDbgTiles] = dw.tiles;
                g_mqa_dbg[kDbgRows] = dw.rows;
                g_mqa_dbg[kDbgChunks] = cur.k + 1;
            }
#endif
        }
        __syncwarp();  // reconverge before the CTA barrier (an aligned barrier)
    } else if (warp < kProdWarp) {
        // ------------------------------------------------------------ epilogue
        const int group = warp >> 2;        // takes tiles i with i % kEpiGroups == group
        const int quarter = warp & 3;       // TMEM lane quarter this warp may access
        const int r = quarter * 32 + lane;  // token within the tile
        const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
        TableCursor cur;
        int qi = -1;
        bool stop = false;
#ifdef MQA_DEBUG
        int walked = 0, taken = 0;
#endif
        while (!stop && cur.next<true>(T, cf, a, lane) == 0) {
            const UnitDesc d = cur.desc(T);
            const int info = cur.info(T);
#ifdef MQA_DEBUG
            ++walked;
#endif
            if (info & 1) {
                if (qi >= 0) {
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(&qempty[qi & 1]);
                }
                qi = info >> 1;
                if (!warp_wait(&qfull[qi & 1], (uint32_t)(qi >> 1) & 1, cf, a, lane)) break;
            }
            const int nt = unit_tiles(d);
            // a unit's two tiles belong to two different groups: at most one is ours
            int k = -1;
            for (int kk = 0; kk < nt; ++kk)
                if ((d.tile + kk) % kEpiGroups == group) k = kk;
            if (k < 0) continue;
            // the token's scale, read from its page now; the load completes while
            // the tile's MMAs run
            const int tu = k * kTile + r;  // token within the unit
            const int t = d.t0 + tu;
            float scale = 0.f;
            if (t < d.ctx) {
                const int p = sh >= 8 ? 0 : (tu >> sh);
                const int row = sh >= 8 ? (d.t0 & (a.page_size - 1)) + tu : tu & (a.page_size - 1);
                int pg = cur.pages(T)[p];
                if (pg < 0 || pg >= a.num_pages) pg = 0;  // as the producer does
                scale = ld_cg_f32(a.kv + (int64_t)pg * a.page_bytes +
                                  (int64_t)a.page_size * D + row * 4);
            }
            const int tile = d.tile + k;
            const int slot = tile & (nacc - 1);
            if (!warp_wait(&accfull[slot], (uint32_t)(tile >> acc_shift) & 1, cf, a, lane)) {
                stop = true;
                break;
            }
            ptx::tc_fence_after();
            float* orow = a.out + ((int64_t)d.b * a.next_n) * a.out_len + t;
            epilogue_tile<H, 64>(lane_base + (uint32_t)(slot * astride), wbuf + (qi & 1) * 256, scale,
                             a.next_n, d.ctx, t, a.out_len, orow, &accempty[slot], lane);
#ifdef MQA_DEBUG
            ++taken;
#endif
        }
#ifdef MQA_DEBUG
        if (lane == 0 && !stop && !cf->abort) {
            g_mqa_dbg[kDbgEpiUnits + warp] = walked;
            g_mqa_dbg[kDbgEpiTiles + warp] = taken;
        }
#endif
    } else if (warp == kTailWarp) {
        // ------------------------------------------------------------ tail fill
        if (a.flags & MQA_FLAG_VALIDATE) check_schedule(a, cta, lane);
        tail_fill(a, cta, 0, 1, lane);
    } else {
        // ------------------------------------------------------------ work table
        build_table(a, cta, T, cf, lane, first, full, qfull, row_bytes, q_bytes, q_load, page_load);
    }

    ptx::tc_fence_before();
    __syncthreads();
#ifdef MQA_DEBUG
    // every role is done: they walked the same units (the builder placed
    // them, the producer and every epilogue warp walked them, the MMA issued
    // them), each epilogue warp took its group's share of the tiles, and each
    // pipeline barrier completed as many phases as it was used
    if (threadIdx.x == 0 && !cf->abort) {
        const int U = g_mqa_dbg[kDbgUnits], TT = g_mqa_dbg[kDbgTiles];
        const int R = g_mqa_dbg[kDbgRows], K = g_mqa_dbg[kDbgChunks];
        bool ok = U >= 0 && TT >= 0 && R >= 0 && K >= 1 && g_mqa_dbg[kDbgBuilt] == U &&
                  g_mqa_dbg[kDbgProd] == U;
        for (int w = 0; w < kProdWarp; ++w)
            ok = ok && g_mqa_dbg[kDbgEpiUnits + w] == U &&
                 g_mqa_dbg[kDbgEpiTiles + w] == debug_share(TT, w >> 2, kEpiGroups);
        for (int s = 0; s < NS; ++s) {
            const int n = debug_share(U, s, NS);
            ok = ok && debug_phases(&full[s], n) && debug_phases(&empty[s], n);
        }
        for (int i = 0; i < nacc; ++i) {
            const int n = debug_share(TT, i, nacc);
            ok = ok && debug_phases(&accfull[i], n) && debug_phases(&accempty[i], n);
        }
        for (int i = 0; i < 2; ++i)
            ok = ok && debug_phases(&qfull[i], debug_share(R, i, 2)) &&
                 debug_phases(&qempty[i], debug_share(R > 0 ? R - 1 : 0, i, 2)) &&
                 debug_phases(&T.full[i], debug_share(K, i, 2)) &&
                 debug_phases(&T.empty[i], debug_share(K, i, 2));
        ok = ok && debug_phases(drain, 1);
        if (!ok) raise_status(a, MQA_STATUS_DEBUG_INVARIANT);
    }
#endif
    if (warp == kMmaWarp) {
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

int launch_fp8_logits(int H, int D, const LaunchSpec& ls, const CUtensorMap& tm_k,
                      const CUtensorMap& tm_q, const KernelArgs& args) {
#define MQA_FP8_CASE(HH, DD)                                                                 \
    case HH * 1000 + DD:                                                                     \
        return launch_instance(&fp8_logits_kernel<HH, DD>, kFp8Threads, ls, tm_k, tm_q, args);
    switch (H * 1000 + D) {
        MQA_FP8_CASE(4, 32) MQA_FP8_CASE(4, 64) MQA_FP8_CASE(4, 128)
        MQA_FP8_CASE(8, 32) MQA_FP8_CASE(8, 64) MQA_FP8_CASE(8, 128)
        MQA_FP8_CASE(16, 32) MQA_FP8_CASE(16, 64) MQA_FP8_CASE(16, 128)
        MQA_FP8_CASE(32, 32) MQA_FP8_CASE(32, 64) MQA_FP8_CASE(32, 128)
        MQA_FP8_CASE(64, 32) MQA_FP8_CASE(64, 64) MQA_FP8_CASE(64, 128)
        MQA_FP8_CASE(128, 32) MQA_FP8_CASE(128, 64) MQA_FP8_CASE(128, 128)
    }
#undef MQA_FP8_CASE
    return (int)cudaErrorInvalidValue;
}

}  // namespace mqa

