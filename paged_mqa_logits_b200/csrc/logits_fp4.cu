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
// One persistent CTA per SM; one pipeline stage is one 256-token schedule unit
// (two 128-token MMA tiles). 18 warps:
//   warps 0-2    producers (see producer_warp), each issuing every third unit
//                of the work table: one tensor copy per page brings the
//                page's packed codes and block scales together (viewed as
//                rows of D bytes, swizzled so the dequant reads are bank-
//                conflict free); a copy costs the SM's tensor-copy engine
//                about the same whatever its size, so one per page rather
//                than one for the codes and one for the scales. Warp 0 also
//                loads each row's bf16 q tile and weights (from the third row
//                on).
//   warp 3       MMA issuer (TMEM owner): tcgen05 kind::f16 with the A operand
//                (dequantised K, 128 tokens x D) in TMEM and q in shared
//                memory; rings of TMEM slots for A and for the accumulators.
//   warps 4-11   epilogue, two groups of four warps taking tiles in turn (tile
//                i goes to group i mod 2).
//   warps 12-15  dequant (both tiles of a unit): thread = token row; e2m1x2 ->
//                f16x2 (hardware cvt), times the block scale (f16x2 multiply,
//                exact), written to TMEM with tcgen05.st (A never goes back
//                through shared memory). At a row's first unit they also
//                convert the row's q in place (bf16 -> f16) and publish its
//                power-of-two exponent, ahead of the MMA.
// The two epilogue groups keep the epilogue (~0.5 us per tile) off the
// critical path; at N = H the tile cost is then set by the MMA instruction
// rate (8 kind::f16 instructions per 128-token tile).
//   warp 16      the -inf tail of every output row past its last tile.
//   warp 17      builds the work table (build_table) and issues the loads of
//                the first ring round and of the first two rows' q.
#include <cuda_runtime.h>

#include <cstdint>
#include "common.cuh"
#include "epilogue.cuh"

namespace mqa {

constexpr int kMmaWarp4 = kProducers;            // 3
constexpr int kEpiWarp4 = kProducers + 1;        // 4..11
constexpr int kEpiGroups4 = 2;
constexpr int kDeqWarp4 = kEpiWarp4 + 4 * kEpiGroups4;  // 12..15
constexpr int kTailWarp4 = kDeqWarp4 + 4;        // 16
constexpr int kBuildWarp4 = kTailWarp4 + 1;      // 17
constexpr int kFp4Threads = 32 * (kBuildWarp4 + 1);
static_assert(kProducers + 1 + 4 * kEpiGroups4 + 4 == kTableUsers, "table users");

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

// TMEM plan: nacc accumulator slots of `astride` columns, then nA A-operand
// slots of D/2 columns (128 lanes x D f16 = D/2 32-bit columns), within 512.
__host__ __device__ inline void fp4_tmem_plan(int D, int npad, int& nacc, int& nA) {
    const int astride = acc_stride(npad);
    nA = 4;
    nacc = (512 - nA * (D / 2)) / astride;
    nacc = nacc >= 8 ? 8 : (nacc >= 4 ? 4 : 2);
}

template <int H, int D>
__global__ void __launch_bounds__(kFp4Threads, 1)
fp4_logits_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_q,
                  const KernelArgs a) {
    constexpr int kRowBytes = D / 2;                 // packed codes per token
    constexpr int kScaleBytes = D / 16;              // block scales per token
    constexpr int kChunks = kRowBytes / 16;          // 16-byte chunks per packed row
    // the page copy's swizzle (128 B for D = 128, 64 B for D = 64): byte offset
    // o within a page slot lives at o ^ (((o >> 7) & kSwzMask) << 4)
    constexpr uint32_t kSwzMask = D >= 128 ? 7u : 3u;
    constexpr int kKSteps = D / 16;                  // MMA K = 16 f16 per instruction
    constexpr int kACols = D / 2;                    // TMEM columns of one A slot

    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int NS = a.num_stages;
    const int npad = a.npad;
    const int astride = acc_stride(npad);
    int nacc, nA;
    fp4_tmem_plan(D, npad, nacc, nA);            // both powers of two
    const int acc_shift = 31 - __clz(nacc);
    const int a_shift = 31 - __clz(nA);
    const Fp4Smem L = fp4_smem_layout(D, npad, NS, a.page_size);
    const uint32_t stage_bytes = L.stage, page_slot = L.page_slot;
    uint8_t* kst = base + L.kst;
    uint8_t* qbuf = base + L.qbuf;
    float* wbuf = reinterpret_cast<float*>(base + L.wbuf);
    uint64_t* full = reinterpret_cast<uint64_t*>(base + L.bars);
    uint64_t* empty = full + NS;
    uint64_t* qfull = empty + NS;
    uint64_t* qready = qfull + 2;
    uint64_t* qempty = qready + 2;
    uint64_t* qmax = qempty + 2;
    uint64_t* drain = qmax + 2;
    uint64_t* tbars = drain + 1;                 // table full[2], empty[2]
    uint64_t* accfull = tbars + 4;
    uint64_t* accempty = accfull + kMaxAccSlots;
    uint64_t* afull = accempty + kMaxAccSlots;
    uint64_t* aempty = afull + kMaxAccSlots;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(base + L.misc);
    volatile CtaFlags* cf = reinterpret_cast<volatile CtaFlags*>(base + L.misc + 8);
    float* red = reinterpret_cast<float*>(base + L.misc + 24);   // [2][4] per-warp |q| maxima
    volatile int32_t* qexp = reinterpret_cast<volatile int32_t*>(base + L.misc + 56);  // [2]
    const Table T = table_view(base + L.table, tbars, a);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int cta = blockIdx.x;
    const uint32_t a_col0 = (uint32_t)(nacc * astride);          // first A slot column
    uint32_t ncols = 32;
    while (ncols < a_col0 + (uint32_t)(nA * kACols)) ncols <<= 1;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            ptx::mbar_init(&full[s], 1);
            ptx::mbar_init(&empty[s], 4);  // the four dequant warps
        }
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(&qfull[i], 1);
            ptx::mbar_init(&qready[i], 4);
            ptx::mbar_init(&qempty[i], 1 + 4 * kEpiGroups4);
            ptx::mbar_init(&qmax[i], 4);
            ptx::mbar_init(&T.full[i], 32);
            ptx::mbar_init(&T.empty[i], kTableUsers);
        }
        for (int i = 0; i < kMaxAccSlots; ++i) {
            ptx::mbar_init(&accfull[i], 1);
            ptx::mbar_init(&accempty[i], 4);
            ptx::mbar_init(&afull[i], 4);
            ptx::mbar_init(&aempty[i], 1);
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
    if (warp == kMmaWarp4) {
        ptx::tmem_alloc(tmem_holder, ncols);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    ptx::griddep_launch_dependents();
    if (warp >= kEpiWarp4 && warp <= kTailWarp4)  // idle at first: warm L2 with the small inputs
        warm_inputs(a, cta, threadIdx.x - 32 * kEpiWarp4, 32 * (kTailWarp4 + 1 - kEpiWarp4));
    ptx::griddep_wait();

    // bf16 q tile + weights of row b into q buffer q; packed K rows + block
    // scales of page p of unit u into stage s
    const uint32_t qbytes = (uint32_t)(npad * D * 2);
    auto q_load = [&](int q, int b) {
        ptx::tma_load_3d(qbuf + q * qbytes, &tm_q, &qfull[q], 0, b * a.hn, 0);
        ptx::bulk_load(wbuf + q * 256, a.weights + (int64_t)b * a.hn, (uint32_t)(a.hn * 4),
                       &qfull[q]);
    };
    auto page_load = [&](int s, int u, int p, int rows, int row_off, int pg) {
        (void)u;
        (void)rows;
        (void)row_off;  // whole pages: a unit never starts inside a page here
        ptx::tma_load_3d(kst + s * stage_bytes + p * page_slot, &tm_k, &full[s], 0, 0, pg);
    };
    const uint32_t row_bytes = (uint32_t)(kRowBytes + kScaleBytes);
    const uint32_t q_bytes = qbytes + (uint32_t)(a.hn * 4);
    const int first = builder_units(a, T, a.num_stages);

    if (warp < kProducers) {
        // ------------------------------------------------------------ producers
        producer_warp<kProducers>(a, T, warp, lane, first, full, empty, qfull, qempty, cf, row_bytes, q_bytes,
                      q_load, page_load);
    } else if (warp == kMmaWarp4) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc = ptx::instr_desc(0, 0, kTile, (uint32_t)npad);  // f16 x f16
            TableCursor cur;
            int qi = -1;
            bool stop = false;
#ifdef MQA_DEBUG
            DebugWalk dw;
            debug_walk_begin(a, cta, dw);
#endif
            while (!stop && cur.next<false>(T, cf, a, 0) == 0) {
                const UnitDesc d = cur.desc(T);
                const int info = cur.info(T);
#ifdef MQA_DEBUG
                debug_check_unit(a, d, info, dw);
#endif
                if (info & 1) {  // a new row: release the previous q, wait for this one
                    if (qi >= 0) ptx::tc_commit(&qempty[qi & 1]);
                    qi = info >> 1;
                    if (!wait_bounded(&qready[qi & 1], (uint32_t)(qi >> 1) & 1, cf, a)) break;
                }
                const uint32_t b_base = ptx::smem_u32(qbuf + (qi & 1) * npad * D * 2);
                const int nt = unit_tiles(d);
                for (int k = 0; k < nt; ++k) {
                    const int tile = d.tile + k;
                    const int slot = tile & (nacc - 1), aslot = tile & (nA - 1);
                    if (!wait_bounded(&accempty[slot], ((uint32_t)(tile >> acc_shift) & 1) ^ 1, cf, a) ||
                        !wait_bounded(&afull[aslot], (uint32_t)(tile >> a_shift) & 1, cf, a)) {
                        stop = true;
                        break;
                    }
                    ptx::tc_fence_after();
                    const uint32_t d_tmem = tmem + (uint32_t)(slot * astride);
                    const uint32_t a_tmem = tmem + a_col0 + (uint32_t)(aslot * kACols);
#pragma unroll
                    for (int kk = 0; kk < kKSteps; ++kk) {
                        const uint32_t b_addr = b_base + (kk >> 2) * npad * 128 + (kk & 3) * 32;
                        ptx::mma_f16_ts(d_tmem, a_tmem + kk * 8,
                                        ptx::smem_desc(b_addr, 0, 1024, ptx::SW_128B), idesc,
                                        kk > 0 ? 1u : 0u);
                    }
                    ptx::tc_commit(&aempty[aslot]);
                    ptx::tc_commit(&accfull[slot]);
                }
            }
            ptx::tc_commit(drain);
            wait_drain(drain, 0, a);
        }
        __syncwarp();  // reconverge before the CTA barrier (an aligned barrier)
    } else if (warp < kDeqWarp4) {
        // ------------------------------------------------------------ epilogue
        const int group = (warp - kEpiWarp4) >> 2;      // takes tiles i with i % 2 == group
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;
        TableCursor cur;
        int qi = -1, qe = 0;
        const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
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
                const int q = qi & 1;
                // the weights land with q; the dequant warps convert q (see
                // there) and publish the row's exponent
                if (!warp_wait(&qfull[q], (qi >> 1) & 1, cf, a, lane)) break;
                if (!warp_wait(&qready[q], (qi >> 1) & 1, cf, a, lane)) break;
                qe = qexp[q];
            }
            const int q = qi & 1;
            const float post = __int_as_float((127 - qe) << 23);  // 2^-qe, exact
            const int nt = unit_tiles(d);
            for (int k = 0; k < nt; ++k) {
                const int tile = d.tile + k;
                if (tile % kEpiGroups4 != group) continue;
                const int slot = tile & (nacc - 1);
                if (!warp_wait(&accfull[slot], (uint32_t)(tile >> acc_shift) & 1, cf, a, lane)) {
                    stop = true;
                    break;
                }
                ptx::tc_fence_after();
                const int t = d.t0 + k * kTile + r;
                float* orow = a.out + ((int64_t)d.b * a.next_n) * a.out_len + t;
                epilogue_tile<H>(lane_base + (uint32_t)(slot * astride), wbuf + q * 256, post,
                                 a.next_n, d.ctx, t, a.out_len, orow, &accempty[slot], lane);
            }
        }
    } else if (warp < kTailWarp4) {
        // ------------------------------------------------------------ dequant
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;       // token row of a tile = TMEM lane
        const int psh = a.ps_shift, pmask = a.page_size - 1;
        const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16) + a_col0;
        // Row qi's q: wait for its load, then convert it in place (bf16 ->
        // f16 of q * 2^e, e from the row's largest |q|) and publish e. Done
        // here, where the row's first unit is met ahead of the MMA, so the
        // MMA does not wait for it at each row start.
        const int dw = warp - kDeqWarp4;                // warp within the dequant group
        const int et = dw * 32 + lane;
        const int nchunk = npad * D * 2 / 16;           // 16-byte chunks of one q buffer
        auto convert_q = [&](int qi) -> bool {
            const int q = qi & 1;
            if (!warp_wait(&qfull[q], (qi >> 1) & 1, cf, a, lane)) return false;
            if (dw == 0 && lane == 0) cf->q_seen = qi + 1;
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
                red[q * 4 + dw] = mx;
                ptx::mbar_arrive(&qmax[q]);
            }
            if (!warp_wait(&qmax[q], (qi >> 1) & 1, cf, a, lane)) return false;
            mx = fmaxf(fmaxf(red[q * 4 + 0], red[q * 4 + 1]),
                       fmaxf(red[q * 4 + 2], red[q * 4 + 3]));
            int qe = 0;
            if (mx > 0.f && mx < __int_as_float(0x7f800000)) qe = 14 - ilogbf(mx);
            if (qe < -100 || qe > 100) {
                // the row's largest |q| lies outside [2^-86, 2^115): its f16
                // image may lose precision or overflow
                if (dw == 0 && lane == 0) raise_status(a, MQA_STATUS_Q_RANGE);
                qe = max(-100, min(100, qe));
            }
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
            if (et == 0) qexp[q] = qe;
            // make the generic-proxy stores visible to the tensor core (async proxy)
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&qready[q]);
            return true;
        };
        TableCursor cur;
        int s = 0;
        uint32_t ph = 0;
        bool stop = false;
        while (!stop && cur.next<true>(T, cf, a, lane) == 0) {
            const UnitDesc d = cur.desc(T);
            const int info = cur.info(T);
            if ((info & 1) && !convert_q(info >> 1)) break;
            if (!warp_wait(&full[s], ph, cf, a, lane)) break;
            if (warp == kDeqWarp4 && lane == 0) {
                cf->consumed = cur.unit(T) + 1;
            }
            const int nt = unit_tiles(d);
            // this thread's row of both tiles, then the stage is free
            uint4 pk[2][kChunks];
            uint32_t scw[2][2] = {{0, 0}, {0, 0}};
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                if (k < nt) {
                    const int tu = k * kTile + r;  // token within the unit
                    const int pp = tu >> psh;       // its page within the unit
                    const int t = tu & pmask;       // and token within that page
                    const uint8_t* page = kst + s * stage_bytes + pp * page_slot;
                    auto swz = [](uint32_t o) { return o ^ (((o >> 7) & kSwzMask) << 4); };
#pragma unroll
                    for (int c = 0; c < kChunks; ++c)
                        pk[k][c] = lds128(page + swz((uint32_t)(t * kRowBytes + c * 16)));
                    const uint32_t so = swz((uint32_t)(a.page_size * kRowBytes + t * kScaleBytes));
                    if constexpr (kScaleBytes == 8) {
                        const uint2 v = lds64(page + so);
                        scw[k][0] = v.x;
                        scw[k][1] = v.y;
                    } else {
                        scw[k][0] = lds32(page + so);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&empty[s]);
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                if (k >= nt) break;
                const int tile = d.tile + k;
                const int aslot = tile & (nA - 1);
                if (!warp_wait(&aempty[aslot], ((uint32_t)(tile >> a_shift) & 1) ^ 1, cf, a, lane)) {
                    stop = true;
                    break;
                }
                ptx::tc_fence_after();
                const uint32_t dst = lane_base + (uint32_t)(aslot * kACols);
#pragma unroll
                for (int c = 0; c < kChunks; ++c) {
                    // chunk c = blocks 2c and 2c+1 (8 packed bytes each); their two
                    // scale bytes are the 16-bit pair (c & 1) of scale word c / 2
                    uint32_t s_lo, s_hi;
                    scales_pair((scw[k][c >> 1] >> ((c & 1) * 16)) & 0xffffu, s_lo, s_hi);
                    uint32_t o[16];
                    uint32_t t4[4];
                    dequant_word(pk[k][c].x, s_lo, t4);
                    o[0] = t4[0]; o[1] = t4[1]; o[2] = t4[2]; o[3] = t4[3];
                    dequant_word(pk[k][c].y, s_lo, t4);
                    o[4] = t4[0]; o[5] = t4[1]; o[6] = t4[2]; o[7] = t4[3];
                    dequant_word(pk[k][c].z, s_hi, t4);
                    o[8] = t4[0]; o[9] = t4[1]; o[10] = t4[2]; o[11] = t4[3];
                    dequant_word(pk[k][c].w, s_hi, t4);
                    o[12] = t4[0]; o[13] = t4[1]; o[14] = t4[2]; o[15] = t4[3];
                    ptx::tmem_st16(dst + c * 16, o);
                }
                ptx::tmem_st_wait();
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(&afull[aslot]);
            }
            if (++s == NS) { s = 0; ph ^= 1; }
        }
    } else if (warp == kTailWarp4) {
        // ------------------------------------------------------------ tail fill
        if (a.flags & MQA_FLAG_VALIDATE) check_schedule(a, cta, lane);
        tail_fill(a, cta, 0, 1, lane);
    } else {
        // ------------------------------------------------------------ work table
        build_table(a, cta, T, cf, lane, first, full, qfull, row_bytes, q_bytes, q_load, page_load);
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp4) {
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

int launch_fp4_logits(int H, int D, const LaunchSpec& ls, const CUtensorMap& tm_k,
                      const CUtensorMap& tm_q, const KernelArgs& args) {
#define MQA_FP4_CASE(HH, DD)                                                                 \
    case HH * 1000 + DD:                                                                     \
        return launch_instance(&fp4_logits_kernel<HH, DD>, kFp4Threads, ls, tm_k, tm_q, args);
    switch (H * 1000 + D) {
        MQA_FP4_CASE(4, 64) MQA_FP4_CASE(4, 128)
        MQA_FP4_CASE(8, 64) MQA_FP4_CASE(8, 128)
        MQA_FP4_CASE(16, 64) MQA_FP4_CASE(16, 128)
        MQA_FP4_CASE(32, 64) MQA_FP4_CASE(32, 128)
        MQA_FP4_CASE(64, 64) MQA_FP4_CASE(64, 128)
        MQA_FP4_CASE(128, 64) MQA_FP4_CASE(128, 128)
    }
#undef MQA_FP4_CASE
    return (int)cudaErrorInvalidValue;
}

}  // namespace mqa

