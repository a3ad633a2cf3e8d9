// FP8 paged MQA logits on sm_100a (the page "[flashinfer] Blackwell 아키텍처를
// 위한 고성능 Paged MQA Logits 커널 도입": introduction, fp8_paged_mqa_logits;
// section 1: persistent TMA + UMMA kernel, zero-length rows skipped in the task
// iterator, epilogue caching sized by register footprint).
//
// One persistent CTA per SM, 7 warps:
//   warp 0      TMA producer. All lanes first stage the context lengths of the
//               CTA's rows into shared memory (cp.async). Lane 0 then streams
//               the block-table entries of the next tiles into a shared ring
//               (cp.async, several tiles ahead, so no page lookup waits on
//               global memory) and per 128-token tile gathers the K rows of
//               the tile's pages (3-D tensor map, swizzled for the MMA) and
//               their fp32 scales (bulk copy) into a ring stage; per row, the
//               q tile and the row's weights.
//   warp 1      MMA issuer (and TMEM owner): acc[t, c] = sum_d k[t,d] q[c,d]
//               with c = n*H + h, as D/32 tcgen05 kind::f8f6f4 instructions
//               (M = 128 tokens, N = H*next_n padded to 16, fp32 in TMEM),
//               double-buffered accumulators.
//   warps 2-5   epilogue: thread = token (its TMEM lane); logit[n] =
//               sum_h w[n,h] * max(s_t * acc[t, nH+h], 0), -inf past the draft
//               context (a select), one coalesced fp32 store per draft row.
//   warp 6      the -inf tail of every output row past its last tile.
// Every wait is bounded (MQA_STATUS_TIMEOUT, never a trap).
#include <cstdint>
#include "common.cuh"
#include "epilogue.cuh"

namespace mqa {

constexpr int kFp8Threads = 224;

__device__ __forceinline__ void wait_drain(uint64_t* bar, uint32_t parity, const KernelArgs& a) {
    const uint64_t t0 = ptx::globaltimer();
    while (!ptx::mbar_try_wait(bar, parity)) {
        if (ptx::globaltimer() - t0 > a.timeout_ns) {
            raise_status(a, MQA_STATUS_TIMEOUT);
            return;
        }
    }
}

template <int H, int D>
__global__ void __launch_bounds__(kFp8Threads, 1)
fp8_logits_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_q,
                  const KernelArgs a) {
    constexpr uint32_t kSwz = D == 128 ? ptx::SW_128B : (D == 64 ? ptx::SW_64B : ptx::SW_32B);
    constexpr uint32_t kSBO = 8 * D;          // bytes between 8-row core-matrix groups
    constexpr int kStageBytes = kTile * D;
    constexpr int kKSteps = D / 32;           // MMA K = 32 e4m3 per instruction

    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int NS = a.num_stages;
    const int npad = a.npad;
    const int astride = acc_stride(npad);
    const Fp8Smem L = fp8_smem_layout(D, npad, NS);
    uint8_t* kst = base + L.kst;
    uint8_t* qbuf = base + L.qbuf;
    float* scales = reinterpret_cast<float*>(base + L.scales);
    float* wbuf = reinterpret_cast<float*>(base + L.wbuf);
    int32_t* rowctx = reinterpret_cast<int32_t*>(base + L.rows);
    int32_t* pring = reinterpret_cast<int32_t*>(base + L.pages);
    uint64_t* full = reinterpret_cast<uint64_t*>(base + L.bars);
    uint64_t* empty = full + NS;
    uint64_t* qfull = empty + NS;
    uint64_t* qempty = qfull + 2;
    uint64_t* accfull = qempty + 2;
    uint64_t* accempty = accfull + 2;
    uint64_t* drain = accempty + 2;
    uint64_t* rows_ready = drain + 1;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(base + L.misc);
    volatile CtaFlags* cf = reinterpret_cast<volatile CtaFlags*>(base + L.misc + 8);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int cta = blockIdx.x;
    uint32_t ncols = 32;
    while (ncols < 2u * astride) ncols <<= 1;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            ptx::mbar_init(&full[s], 1);
            ptx::mbar_init(&empty[s], 1 + 4);
        }
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(&qfull[i], 1);
            ptx::mbar_init(&qempty[i], 1 + 4);
            ptx::mbar_init(&accfull[i], 1);
            ptx::mbar_init(&accempty[i], 4);
        }
        ptx::mbar_init(drain, 1);
        ptx::mbar_init(rows_ready, 32);
        cf->abort = 0;
        ptx::fence_mbar_init();
        ptx::prefetch_tmap(&tm_k);
        ptx::prefetch_tmap(&tm_q);
    }
    if (warp == 1) {
        ptx::tmem_alloc(tmem_holder, ncols);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    ptx::griddep_launch_dependents();
    ptx::griddep_wait();  // inputs (schedule, context_lens, ...) may come from the previous kernel

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        const RowCache rc = stage_rows(a, cta, rowctx, rows_ready, lane);
        if (lane == 0) {
            const bool ok = wait_bounded(rows_ready, 0, cf, a);
            TileIter it;
            it.init(a, cta, rc);
            TileIter fit = it;  // runs kPageLookahead tiles ahead, fetching page indices
            int fpos = 0, cpos = 0;
            auto fetch_next = [&]() {
                if (fit.valid(a)) {
                    const TilePages tp = tile_pages(fit, a.page_size);
                    const int32_t* src = a.block_table + (int64_t)fit.b * a.max_pages + tp.pfirst;
                    for (int p = 0; p < tp.npg; ++p)
                        ptx::cp_async_4(pring + ((fpos + p) & (kPageRing - 1)), src + p);
                    fpos += tp.npg;
                    fit.next(a);
                }
                ptx::cp_async_commit();
            };
#pragma unroll 1
            for (int i = 0; i < kPageLookahead; ++i) fetch_next();

            int prev_b = -1, qi = -1, s = 0, dropped = -1;
            uint32_t ph = 0;
            const bool inject = (a.flags & MQA_FLAG_TEST_DROP_ARRIVE) != 0;
            while (ok && it.valid(a)) {
                if (it.b != prev_b) {
                    ++qi;
                    const int q = qi & 1;
                    if (!wait_bounded(&qempty[q], ((qi >> 1) & 1) ^ 1, cf, a)) { --qi; break; }
                    ptx::mbar_arrive_expect_tx(&qfull[q], (uint32_t)(npad * D + a.hn * 4));
                    ptx::tma_load_2d(qbuf + q * npad * D, &tm_q, &qfull[q], 0, it.b * a.hn);
                    ptx::bulk_load(wbuf + q * 256, a.weights + (int64_t)it.b * a.hn,
                                   (uint32_t)(a.hn * 4), &qfull[q]);
                    prev_b = it.b;
                }
                if (!wait_bounded(&empty[s], ph ^ 1, cf, a)) break;
                const TilePages tp = tile_pages(it, a.page_size);
                ptx::cp_async_wait<kPageLookahead - 1>();  // this tile's page indices landed
                if (inject && it.idx == 1 && dropped < 0) {
                    dropped = it.idx;  // test only: this stage is never filled
                } else {
                    ptx::mbar_arrive_expect_tx(&full[s], (uint32_t)(tp.npg * tp.rows * (D + 4)));
                    for (int p = 0; p < tp.npg; ++p) {
                        int pg = pring[(cpos + p) & (kPageRing - 1)];
                        if (pg < 0 || pg >= a.num_pages) {
                            if (a.flags & MQA_FLAG_VALIDATE) raise_status(a, MQA_STATUS_BAD_PAGE);
                            pg = 0;  // stay in bounds; the tile's values are then meaningless
                        }
                        ptx::tma_load_3d(kst + s * kStageBytes + p * tp.rows * D, &tm_k, &full[s],
                                         0, tp.row_off, pg);
                        ptx::bulk_load(scales + s * kTile + p * tp.rows,
                                       a.kv + (int64_t)pg * a.page_bytes +
                                           (int64_t)a.page_size * D + tp.row_off * 4,
                                       (uint32_t)(tp.rows * 4), &full[s]);
                    }
                }
                cpos += tp.npg;
                fetch_next();
                if (++s == NS) { s = 0; ph ^= 1; }
                it.next(a);
            }
            ptx::cp_async_wait<0>();
            // Drain: wait (bounded) for every copy this thread issued to land.
            const int n = it.idx;
            for (int i = max(0, n - NS); i < n; ++i)
                if (i != dropped) wait_drain(&full[i % NS], (uint32_t)((i / NS) & 1), a);
            for (int r = max(0, qi - 1); r <= qi; ++r)
                wait_drain(&qfull[r & 1], (uint32_t)((r >> 1) & 1), a);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc = ptx::instr_desc(0, 0, kTile, (uint32_t)npad);
            const bool ok = wait_bounded(rows_ready, 0, cf, a);
            TileIter it;
            it.init(a, cta, row_cache_view(a, cta, rowctx));
            int prev_b = -1, qi = -1, s = 0;
            uint32_t ph = 0;
            while (ok && it.valid(a)) {
                if (it.b != prev_b) {
                    if (prev_b >= 0) ptx::tc_commit(&qempty[qi & 1]);
                    ++qi;
                    if (!wait_bounded(&qfull[qi & 1], (qi >> 1) & 1, cf, a)) break;
                    prev_b = it.b;
                }
                const int acc = it.idx & 1;
                const uint32_t use = (uint32_t)(it.idx >> 1);
                if (!wait_bounded(&accempty[acc], (use & 1) ^ 1, cf, a)) break;
                if (!wait_bounded(&full[s], ph, cf, a)) break;
                ptx::tc_fence_after();
                const uint32_t d_tmem = tmem + (uint32_t)(acc * astride);
                const uint32_t a_base = ptx::smem_u32(kst + s * kStageBytes);
                const uint32_t b_base = ptx::smem_u32(qbuf + (qi & 1) * npad * D);
#pragma unroll
                for (int kk = 0; kk < kKSteps; ++kk) {
                    ptx::mma_f8f6f4_ss(d_tmem, ptx::smem_desc(a_base + kk * 32, 0, kSBO, kSwz),
                                       ptx::smem_desc(b_base + kk * 32, 0, kSBO, kSwz), idesc,
                                       kk > 0 ? 1u : 0u);
                }
                ptx::tc_commit(&empty[s]);
                ptx::tc_commit(&accfull[acc]);
                if (++s == NS) { s = 0; ph ^= 1; }
                it.next(a);
            }
            // all MMAs issued by this thread are complete before TMEM is freed
            ptx::tc_commit(drain);
            wait_drain(drain, 0, a);
        }
    } else if (warp < 6) {
        // ------------------------------------------------------------ epilogue
        const int quarter = warp & 3;       // TMEM lane quarter this warp may access
        const int r = quarter * 32 + lane;  // token within the tile
        const bool ok = wait_bounded(rows_ready, 0, cf, a);
        TileIter it;
        it.init(a, cta, row_cache_view(a, cta, rowctx));
        int prev_b = -1, qi = -1, s = 0;
        const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
        while (ok && it.valid(a)) {
            if (it.b != prev_b) {
                if (prev_b >= 0) {
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(&qempty[qi & 1]);
                }
                ++qi;
                if (!wait_bounded(&qfull[qi & 1], (qi >> 1) & 1, cf, a)) break;
                prev_b = it.b;
            }
            const int acc = it.idx & 1;
            const uint32_t use = (uint32_t)(it.idx >> 1);
            if (!wait_bounded(&accfull[acc], use & 1, cf, a)) break;
            ptx::tc_fence_after();
            const float scale = scales[s * kTile + r];
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&empty[s]);
            const int t = it.t0() + r;
            float* orow = a.out + ((int64_t)it.b * a.next_n) * a.out_len + t;
            epilogue_tile<H, true>(lane_base + (uint32_t)(acc * astride), wbuf + (qi & 1) * 256,
                                   scale, 1.f, a.next_n, it.ctx, t, a.out_len, orow,
                                   &accempty[acc], lane);
            if (++s == NS) s = 0;
            it.next(a);
        }
    } else {
        // ------------------------------------------------------------ tail fill
        if (a.flags & MQA_FLAG_VALIDATE) check_schedule(a, cta, lane);
        tail_fill(a, cta, 0, 1, lane);
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, ncols);
    }
}

// Explicit instantiations: H in {4, 8, 16, 32, 64, 128}, D in {32, 64, 128}.
#define MQA_FP8_INST(H, D)                                                                \
    template __global__ void fp8_logits_kernel<H, D>(const __grid_constant__ CUtensorMap, \
                                                     const __grid_constant__ CUtensorMap, \
                                                     const KernelArgs);
#define MQA_FP8_INST_D(H) MQA_FP8_INST(H, 32) MQA_FP8_INST(H, 64) MQA_FP8_INST(H, 128)
MQA_FP8_INST_D(4)
MQA_FP8_INST_D(8)
MQA_FP8_INST_D(16)
MQA_FP8_INST_D(32)
MQA_FP8_INST_D(64)
MQA_FP8_INST_D(128)

}  // namespace mqa
