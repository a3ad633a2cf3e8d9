// FP4 paged MQA logits on sm_100a (the page "[flashinfer] Blackwell 아키텍처를
// 위한 고성능 Paged MQA Logits 커널 도입": introduction, fp4_paged_mqa_logits).
//
// K is stored as e2m1 codes (two per byte) with one e4m3 scale per 16
// elements; q is bf16. The block-scaled product must happen inside the dot
// product, and a bf16 q cannot be expressed in a block-scaled FP4 MMA, so K is
// dequantised on the fly: code * scale has at most 6 significant bits and
// lies in [2^-10, 2688], so it is EXACT in f16. q is brought to f16 with one
// power-of-two scale 2^e per batch row (largest |q| of the row mapped into
// [2^14, 2^15)); the epilogue multiplies each logit by 2^-e, which undoes the
// scale exactly. The conversion of q is exact unless a nonzero |q| is below
// about 2^-31 of its row's largest magnitude.
//
// One persistent CTA per SM, 10 warps:
//   warp 0      TMA producer: packed K rows of a 128-token tile (3-D tensor
//               map, swizzled so the dequant reads are bank-conflict free),
//               the block scales (bulk copy); per row, the bf16 q tile and
//               the weights.
//   warp 1      MMA issuer (TMEM owner): tcgen05 kind::f16 with the A operand
//               (dequantised K, 128 tokens x D) in TMEM and q in shared
//               memory; double-buffered A and accumulators.
//   warps 2-5   epilogue, and per row the in-place q conversion bf16 -> f16.
//   warps 6-9   dequant: thread = token row; e2m1x2 -> f16x2 (hardware cvt),
//               times the block scale (f16x2 multiply, exact), written to TMEM
//               with tcgen05.st (no shared-memory round trip for A).
//   warp 10     the -inf tail of every output row past its last tile.
// The producer stages row context lengths and streams block-table entries
// ahead of use exactly as the FP8 kernel does.
#include <cstdint>
#include "common.cuh"
#include "epilogue.cuh"

namespace mqa {

constexpr int kFp4Threads = 352;

__device__ __forceinline__ void wait_drain4(uint64_t* bar, uint32_t parity, const KernelArgs& a) {
    const uint64_t t0 = ptx::globaltimer();
    while (!ptx::mbar_try_wait(bar, parity)) {
        if (ptx::globaltimer() - t0 > a.timeout_ns) {
            raise_status(a, MQA_STATUS_TIMEOUT);
            return;
        }
    }
}

__device__ __forceinline__ uint32_t lds32(const void* p) {
    uint32_t v;
    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(ptx::smem_u32(p)));
    return v;
}

__device__ __forceinline__ uint2 lds64(const void* p) {
    uint2 v;
    asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(ptx::smem_u32(p)));
    return v;
}

__device__ __forceinline__ uint4 lds128(const void* p) {
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(ptx::smem_u32(p)));
    return v;
}

// Four packed bytes (eight e2m1 codes) -> four f16x2 words, each times the
// f16x2 block scale `s2` (the same scale in both halves). Element order is
// kept: the low nibble of byte j goes to the low half of word j.
__device__ __forceinline__ void dequant_word(uint32_t w, uint32_t s2, uint32_t (&o)[4]) {
    uint32_t c0, c1, c2, c3;
    asm volatile(
        "{\n\t.reg .b8 b0, b1, b2, b3;\n\tmov.b32 {b0, b1, b2, b3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\tcvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, b2;\n\tcvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
        : "=r"(c0), "=r"(c1), "=r"(c2), "=r"(c3) : "r"(w));
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(o[0]) : "r"(c0), "r"(s2));
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(o[1]) : "r"(c1), "r"(s2));
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(o[2]) : "r"(c2), "r"(s2));
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(o[3]) : "r"(c3), "r"(s2));
}

// Two e4m3 scales (a 16-bit pair) -> f16x2, then each replicated into both
// halves: lo gets scale 0, hi gets scale 1.
__device__ __forceinline__ void scales_pair(uint32_t two, uint32_t& lo, uint32_t& hi) {
    uint32_t s;
    asm("{\n\t.reg .b16 h;\n\tcvt.u16.u32 h, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, h;\n\t}"
        : "=r"(s) : "r"(two));
    lo = __byte_perm(s, s, 0x1010);
    hi = __byte_perm(s, s, 0x3232);
}

// bf16 bits -> f16 bits of (x * 2^e), round to nearest even.
__device__ __forceinline__ uint32_t bf16x2_to_f16x2_scaled(uint32_t v, float scale) {
    const float lo = __uint_as_float(v << 16) * scale;
    const float hi = __uint_as_float(v & 0xffff0000u) * scale;
    uint32_t r;
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

template <int H, int D>
__global__ void __launch_bounds__(kFp4Threads, 1)
fp4_logits_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_q,
                  const KernelArgs a) {
    constexpr int kRowBytes = D / 2;                 // packed codes per token
    constexpr int kScaleBytes = D / 16;              // block scales per token
    constexpr int kStageBytes = kTile * kRowBytes;
    constexpr int kChunks = kRowBytes / 16;          // 16-byte chunks per packed row
    constexpr uint32_t kSwzMask = kRowBytes == 64 ? 3u : 1u;  // TMA SW64 / SW32 pattern
    constexpr uint32_t kSwzShift = kRowBytes == 64 ? 1u : 2u;
    constexpr int kKSteps = D / 16;                  // MMA K = 16 f16 per instruction
    constexpr int kACols = D / 2;                    // TMEM columns of one A buffer

    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int NS = a.num_stages;
    const int npad = a.npad;
    const int astride = acc_stride(npad);
    const Fp4Smem L = fp4_smem_layout(D, npad, NS);
    uint8_t* kst = base + L.kst;
    uint8_t* qbuf = base + L.qbuf;
    uint8_t* sc = base + L.scales;
    float* wbuf = reinterpret_cast<float*>(base + L.wbuf);
    int32_t* rowctx = reinterpret_cast<int32_t*>(base + L.rows);
    int32_t* pring = reinterpret_cast<int32_t*>(base + L.pages);
    uint64_t* full = reinterpret_cast<uint64_t*>(base + L.bars);
    uint64_t* empty = full + NS;
    uint64_t* qfull = empty + NS;
    uint64_t* qready = qfull + 2;
    uint64_t* qempty = qready + 2;
    uint64_t* afull = qempty + 2;
    uint64_t* aempty = afull + 2;
    uint64_t* accfull = aempty + 2;
    uint64_t* accempty = accfull + 2;
    uint64_t* qmax = accempty + 2;
    uint64_t* drain = qmax + 2;
    uint64_t* rows_ready = drain + 1;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(base + L.misc);
    volatile CtaFlags* cf = reinterpret_cast<volatile CtaFlags*>(base + L.misc + 4);
    float* red = reinterpret_cast<float*>(base + L.misc + 8);    // [2][4] per-warp |q| maxima

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int cta = blockIdx.x;
    const uint32_t a_col0 = 2u * astride;                         // first A buffer column
    uint32_t ncols = 32;
    while (ncols < a_col0 + 2u * kACols) ncols <<= 1;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            ptx::mbar_init(&full[s], 1);
            ptx::mbar_init(&empty[s], 4);
        }
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(&qfull[i], 1);
            ptx::mbar_init(&qready[i], 4);
            ptx::mbar_init(&qempty[i], 1 + 4);
            ptx::mbar_init(&afull[i], 4);
            ptx::mbar_init(&aempty[i], 1);
            ptx::mbar_init(&accfull[i], 1);
            ptx::mbar_init(&accempty[i], 4);
            ptx::mbar_init(&qmax[i], 4);
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
    ptx::griddep_wait();

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
            const uint32_t qbytes = (uint32_t)(npad * D * 2);
            while (ok && it.valid(a)) {
                if (it.b != prev_b) {
                    ++qi;
                    const int q = qi & 1;
                    if (!wait_bounded(&qempty[q], ((qi >> 1) & 1) ^ 1, cf, a)) { --qi; break; }
                    ptx::mbar_arrive_expect_tx(&qfull[q], qbytes + (uint32_t)(a.hn * 4));
                    ptx::tma_load_3d(qbuf + q * qbytes, &tm_q, &qfull[q], 0, it.b * a.hn, 0);
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
                    ptx::mbar_arrive_expect_tx(
                        &full[s], (uint32_t)(tp.npg * tp.rows * (kRowBytes + kScaleBytes)));
                    for (int p = 0; p < tp.npg; ++p) {
                        int pg = pring[(cpos + p) & (kPageRing - 1)];
                        if (pg < 0 || pg >= a.num_pages) {
                            if (a.flags & MQA_FLAG_VALIDATE) raise_status(a, MQA_STATUS_BAD_PAGE);
                            pg = 0;
                        }
                        ptx::tma_load_3d(kst + s * kStageBytes + p * tp.rows * kRowBytes, &tm_k,
                                         &full[s], 0, tp.row_off, pg);
                        ptx::bulk_load(sc + (s * kTile + p * tp.rows) * kScaleBytes,
                                       a.kv + (int64_t)pg * a.page_bytes +
                                           (int64_t)a.page_size * kRowBytes +
                                           tp.row_off * kScaleBytes,
                                       (uint32_t)(tp.rows * kScaleBytes), &full[s]);
                    }
                }
                cpos += tp.npg;
                fetch_next();
                if (++s == NS) { s = 0; ph ^= 1; }
                it.next(a);
            }
            ptx::cp_async_wait<0>();
            const int n = it.idx;
            for (int i = max(0, n - NS); i < n; ++i)
                if (i != dropped) wait_drain4(&full[i % NS], (uint32_t)((i / NS) & 1), a);
            for (int r = max(0, qi - 1); r <= qi; ++r)
                wait_drain4(&qfull[r & 1], (uint32_t)((r >> 1) & 1), a);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc = ptx::instr_desc(0, 0, kTile, (uint32_t)npad);  // f16 x f16
            const bool ok = wait_bounded(rows_ready, 0, cf, a);
            TileIter it;
            it.init(a, cta, row_cache_view(a, cta, rowctx));
            int prev_b = -1, qi = -1;
            while (ok && it.valid(a)) {
                if (it.b != prev_b) {
                    if (prev_b >= 0) ptx::tc_commit(&qempty[qi & 1]);
                    ++qi;
                    if (!wait_bounded(&qready[qi & 1], (qi >> 1) & 1, cf, a)) break;
                    prev_b = it.b;
                }
                const int acc = it.idx & 1;
                const uint32_t use = (uint32_t)(it.idx >> 1);
                if (!wait_bounded(&accempty[acc], (use & 1) ^ 1, cf, a)) break;
                if (!wait_bounded(&afull[acc], use & 1, cf, a)) break;
                ptx::tc_fence_after();
                const uint32_t d_tmem = tmem + (uint32_t)(acc * astride);
                const uint32_t a_tmem = tmem + a_col0 + (uint32_t)(acc * kACols);
                const uint32_t b_base = ptx::smem_u32(qbuf + (qi & 1) * npad * D * 2);
#pragma unroll
                for (int kk = 0; kk < kKSteps; ++kk) {
                    const uint32_t b_addr = b_base + (kk >> 2) * npad * 128 + (kk & 3) * 32;
                    ptx::mma_f16_ts(d_tmem, a_tmem + kk * 8,
                                    ptx::smem_desc(b_addr, 0, 1024, ptx::SW_128B), idesc,
                                    kk > 0 ? 1u : 0u);
                }
                ptx::tc_commit(&aempty[acc]);
                ptx::tc_commit(&accfull[acc]);
                it.next(a);
            }
            ptx::tc_commit(drain);
            wait_drain4(drain, 0, a);
        }
    } else if (warp < 6) {
        // ------------------------------------------------------------ epilogue (+ q conversion)
        const int ew = warp - 2;          // 0..3
        const int et = threadIdx.x - 64;  // 0..127
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;
        const bool ok = wait_bounded(rows_ready, 0, cf, a);
        TileIter it;
        it.init(a, cta, row_cache_view(a, cta, rowctx));
        int prev_b = -1, qi = -1, qe = 0;
        const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
        const int nchunk = npad * D * 2 / 16;        // 16-byte chunks of one q buffer
        while (ok && it.valid(a)) {
            if (it.b != prev_b) {
                if (prev_b >= 0) {
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(&qempty[qi & 1]);
                }
                ++qi;
                const int q = qi & 1;
                if (!wait_bounded(&qfull[q], (qi >> 1) & 1, cf, a)) break;
                // in-place q conversion: bf16 -> f16 of q * 2^e
                uint8_t* qb = qbuf + q * npad * D * 2;
                float mx = 0.f;
                for (int c = et; c < nchunk; c += 128) {
                    const int row = (c * 16 / 128) % npad;
                    if (row < a.hn) {
                        const uint4 v = lds128(qb + c * 16);
                        const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                        for (int x = 0; x < 4; ++x) {
                            mx = fmaxf(mx, fabsf(__uint_as_float(u[x] << 16)));
                            mx = fmaxf(mx, fabsf(__uint_as_float(u[x] & 0xffff0000u)));
                        }
                    }
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
                if (lane == 0) {
                    red[q * 4 + ew] = mx;
                    ptx::mbar_arrive(&qmax[q]);
                }
                if (!wait_bounded(&qmax[q], (qi >> 1) & 1, cf, a)) break;
                mx = fmaxf(fmaxf(red[q * 4 + 0], red[q * 4 + 1]),
                           fmaxf(red[q * 4 + 2], red[q * 4 + 3]));
                qe = 0;
                if (mx > 0.f && mx < __int_as_float(0x7f800000)) qe = 14 - ilogbf(mx);
                qe = max(-100, min(100, qe));
                const float up = __int_as_float((127 + qe) << 23);  // 2^qe, exact
                for (int c = et; c < nchunk; c += 128) {
                    const int row = (c * 16 / 128) % npad;
                    uint4 o = make_uint4(0, 0, 0, 0);
                    if (row < a.hn) {
                        const uint4 v = lds128(qb + c * 16);
                        o.x = bf16x2_to_f16x2_scaled(v.x, up);
                        o.y = bf16x2_to_f16x2_scaled(v.y, up);
                        o.z = bf16x2_to_f16x2_scaled(v.z, up);
                        o.w = bf16x2_to_f16x2_scaled(v.w, up);
                    }
                    *reinterpret_cast<uint4*>(qb + c * 16) = o;
                }
                // make the generic-proxy stores visible to the tensor core (async proxy)
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(&qready[q]);
                prev_b = it.b;
            }
            const int acc = it.idx & 1;
            const uint32_t use = (uint32_t)(it.idx >> 1);
            if (!wait_bounded(&accfull[acc], use & 1, cf, a)) break;
            ptx::tc_fence_after();
            const int q = qi & 1;
            const float post = __int_as_float((127 - qe) << 23);  // 2^-qe, exact
            const int t = it.t0() + r;
            float* orow = a.out + ((int64_t)it.b * a.next_n) * a.out_len + t;
            epilogue_tile<H, false>(lane_base + (uint32_t)(acc * astride), wbuf + q * 256, 1.f,
                                    post, a.next_n, it.ctx, t, a.out_len, orow, &accempty[acc],
                                    lane);
            it.next(a);
        }
    } else if (warp < 10) {
        // ------------------------------------------------------------ dequant
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;     // token row of the tile = TMEM lane
        const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16) + a_col0;
        const bool ok = wait_bounded(rows_ready, 0, cf, a);
        TileIter it;
        it.init(a, cta, row_cache_view(a, cta, rowctx));
        int s = 0;
        uint32_t ph = 0;
        while (ok && it.valid(a)) {
            if (!wait_bounded(&full[s], ph, cf, a)) break;
            const uint8_t* row = kst + s * kStageBytes + r * kRowBytes;
            uint4 pk[kChunks];
#pragma unroll
            for (int c = 0; c < kChunks; ++c)
                pk[c] = lds128(row + ((c ^ ((r >> kSwzShift) & kSwzMask)) << 4));
            uint32_t scw[2];
            if constexpr (kScaleBytes == 8) {
                const uint2 v = lds64(sc + (s * kTile + r) * kScaleBytes);
                scw[0] = v.x;
                scw[1] = v.y;
            } else {
                scw[0] = lds32(sc + (s * kTile + r) * kScaleBytes);
                scw[1] = 0;
            }
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&empty[s]);

            const int ab = it.idx & 1;
            const uint32_t use = (uint32_t)(it.idx >> 1);
            if (!wait_bounded(&aempty[ab], (use & 1) ^ 1, cf, a)) break;
            ptx::tc_fence_after();
            const uint32_t dst = lane_base + (uint32_t)(ab * kACols);
#pragma unroll
            for (int c = 0; c < kChunks; ++c) {
                // chunk c = blocks 2c and 2c+1 (8 packed bytes each); their two
                // scale bytes are the 16-bit pair (c & 1) of scale word c / 2
                uint32_t s_lo, s_hi;
                scales_pair((scw[c >> 1] >> ((c & 1) * 16)) & 0xffffu, s_lo, s_hi);
                uint32_t o[16];
                uint32_t t4[4];
                const uint32_t words[4] = {pk[c].x, pk[c].y, pk[c].z, pk[c].w};
                dequant_word(words[0], s_lo, t4);
                o[0] = t4[0]; o[1] = t4[1]; o[2] = t4[2]; o[3] = t4[3];
                dequant_word(words[1], s_lo, t4);
                o[4] = t4[0]; o[5] = t4[1]; o[6] = t4[2]; o[7] = t4[3];
                dequant_word(words[2], s_hi, t4);
                o[8] = t4[0]; o[9] = t4[1]; o[10] = t4[2]; o[11] = t4[3];
                dequant_word(words[3], s_hi, t4);
                o[12] = t4[0]; o[13] = t4[1]; o[14] = t4[2]; o[15] = t4[3];
                ptx::tmem_st16(dst + c * 16, o);
            }
            ptx::tmem_st_wait();
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&afull[ab]);
            if (++s == NS) { s = 0; ph ^= 1; }
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

#define MQA_FP4_INST(H, D)                                                                \
    template __global__ void fp4_logits_kernel<H, D>(const __grid_constant__ CUtensorMap, \
                                                     const __grid_constant__ CUtensorMap, \
                                                     const KernelArgs);
#define MQA_FP4_INST_D(H) MQA_FP4_INST(H, 64) MQA_FP4_INST(H, 128)
MQA_FP4_INST_D(4)
MQA_FP4_INST_D(8)
MQA_FP4_INST_D(16)
MQA_FP4_INST_D(32)
MQA_FP4_INST_D(64)
MQA_FP4_INST_D(128)

}  // namespace mqa
