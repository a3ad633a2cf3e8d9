// Device-side pieces shared by the logits kernels: the argument block, shared
// memory layouts, the bounded pipeline wait, the work iterator every warp role
// runs, the producer warp, the -inf tail fill and the validate-mode schedule
// check.
#pragma once
#include <cstdint>
#include "ptx.cuh"
#include "mqa_logits.h"

namespace mqa {

constexpr int kUnit = MQA_SCHEDULE_UNIT;  // tokens per schedule unit = one pipeline stage
constexpr int kTile = 128;                // tokens per MMA tile (M = 128)
constexpr int kTilesPerUnit = kUnit / kTile;
constexpr int kRowCache = 1024;           // context lengths of a CTA's rows staged in shared memory
constexpr int kMaxUnitPages = 32;         // pages per unit at the smallest page size (8)
constexpr int kProducers = 3;             // producer warps; warp p issues units p, p + 3, ...
constexpr int kPageLookahead = 3;         // own units whose block-table entries are fetched ahead
constexpr int kPageRingUnits = 16;        // >= kProducers * (kPageLookahead + 1)
constexpr int kPageRing = kPageRingUnits * kMaxUnitPages;
constexpr int kMaxAccSlots = 8;           // TMEM accumulator slots (tiles in flight)
constexpr int kScaleRing = 16;            // units of per-token scales held (FP8): see producer_warp

// Everything a logits kernel needs besides its tensor maps (by value).
struct KernelArgs {
    const uint8_t* kv;
    const int32_t* block_table;
    const int32_t* context_lens;
    const float* weights;
    const int32_t* schedule;
    float* out;
    int32_t* status;
    int64_t page_bytes;       // bytes per KV page
    int32_t batch, next_n, heads, head_dim, page_size, num_pages, max_pages, out_len;
    int32_t num_ctas;         // schedule length - 1
    int32_t hn;               // heads * next_n
    int32_t npad;             // hn rounded up to 16: MMA N
    int32_t num_stages;       // K ring depth (units)
    int32_t ctx_cap;          // min(out_len, max_pages * page_size)
    int32_t ps_shift;         // log2(page_size)
    uint32_t flags;
    uint64_t timeout_ns;
};

__host__ __device__ inline int acc_stride(int npad) { return npad < 32 ? 32 : npad; }

// Shared-memory layout of the FP8 kernel: byte offsets from the 1024-aligned
// dynamic shared memory base. Used by the kernel and by the launcher.
struct Fp8Smem {
    uint32_t kst, qbuf, scales, wbuf, rows, pages, bars, misc, total;
};

__host__ __device__ inline Fp8Smem fp8_smem_layout(int D, int npad, int stages) {
    Fp8Smem L;
    uint32_t off = 0;
    L.kst = off;                                  // stages x [256 tokens][D] e4m3, swizzled
    off += (uint32_t)stages * kUnit * D;
    L.qbuf = off;                                 // 2 x [npad][D] e4m3, swizzled
    off += 2u * npad * D;
    off = (off + 1023) & ~1023u;
    L.scales = off;                               // kScaleRing x [256] fp32 (a ring of its own)
    off += (uint32_t)kScaleRing * kUnit * 4;
    L.wbuf = off;                                 // 2 x [256] fp32 weights
    off += 2u * 256 * 4;
    L.rows = off;                                 // [kRowCache] context lengths
    off += kRowCache * 4;
    L.pages = off;                                // [kPageRing] block-table entries
    off += kPageRing * 4;
    L.bars = off;                                 // 2*stages + 6 + 2*kMaxAccSlots mbarriers
                                                  // (K stages are released by the MMA)
    off += (uint32_t)(2 * stages + 6 + 2 * kMaxAccSlots) * 8;
    L.misc = off;                                 // TMEM address, abort flag
    off += 16;
    L.total = off + 1024;                         // slack for aligning the base
    return L;
}

// Shared-memory layout of the FP4 kernel.
struct Fp4Smem {
    uint32_t kst, qbuf, scales, wbuf, rows, pages, bars, misc, total;
};

__host__ __device__ inline Fp4Smem fp4_smem_layout(int D, int npad, int stages) {
    Fp4Smem L;
    uint32_t off = 0;
    L.kst = off;                                  // stages x [256 tokens][D/2] packed e2m1, swizzled
    off += (uint32_t)stages * kUnit * (D / 2);
    off = (off + 1023) & ~1023u;
    L.qbuf = off;                                 // 2 x [D/64][npad][64] bf16 -> f16 in place
    off += 2u * npad * D * 2;
    L.scales = off;                               // stages x [256][D/16] e4m3 block scales
    off += (uint32_t)stages * kUnit * (D / 16);
    off = (off + 15) & ~15u;
    L.wbuf = off;                                 // 2 x [256] fp32 weights
    off += 2u * 256 * 4;
    L.rows = off;                                 // [kRowCache] context lengths
    off += kRowCache * 4;
    L.pages = off;                                // [kPageRing] block-table entries
    off += kPageRing * 4;
    L.bars = off;                                 // 2*stages + 10 + 4*kMaxAccSlots mbarriers
    off += (uint32_t)(2 * stages + 10 + 4 * kMaxAccSlots) * 8;
    L.misc = off;                                 // TMEM address, abort flag, q maxima
    off += 48;
    L.total = off + 1024;
    return L;
}

// Host side of a logits launch: each kernel file dispatches over its
// compiled (H, D) instances and launches with these settings.
struct LaunchSpec {
    int grid;
    uint32_t smem;
    void* stream;
    bool pdl;
};

// Returns cudaSuccess, or cudaErrorInvalidValue when no instance matches
// (H, D); other codes come from the CUDA runtime.
int launch_fp8_logits(int H, int D, const LaunchSpec& ls, const CUtensorMap& tm_k,
                      const CUtensorMap& tm_q, const KernelArgs& args);
int launch_fp4_logits(int H, int D, const LaunchSpec& ls, const CUtensorMap& tm_k,
                      const CUtensorMap& tm_q, const KernelArgs& args);

// Shared across the CTA: set once any role gives up.
struct CtaFlags {
    int32_t abort;
};

// Optional timeline tracing for development builds (-DMQA_TRACE): per-CTA
// globaltimer stamps at fixed slots of a device array.
#ifdef MQA_TRACE
static __device__ unsigned long long g_mqa_trace[4096 * 64];
#define MQA_TRACE_AT(slot) (g_mqa_trace[blockIdx.x * 64 + (slot)] = ptx::globaltimer())
#define MQA_TRACE_VAL(slot, v) (g_mqa_trace[blockIdx.x * 64 + (slot)] = (unsigned long long)(v))
#else
#define MQA_TRACE_AT(slot) ((void)0)
#define MQA_TRACE_VAL(slot, v) ((void)0)
#endif

__device__ __forceinline__ void raise_status(const KernelArgs& a, uint32_t bits) {
    if (a.status != nullptr) atomicOr(reinterpret_cast<uint32_t*>(a.status), bits);
}

// Waits for phase `parity` of `bar` to complete. Returns false if the CTA was
// aborted by another role or if the wait exceeded the timeout (then the
// status word gets MQA_STATUS_TIMEOUT and the CTA is aborted). Never traps.
__device__ __forceinline__ bool wait_bounded(uint64_t* bar, uint32_t parity,
                                             volatile CtaFlags* cf, const KernelArgs& a) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = ptx::globaltimer();
    while (true) {
        if (ptx::mbar_try_wait(bar, parity)) return true;
        if (cf->abort) return false;
        if (ptx::globaltimer() - t0 > a.timeout_ns) {
            raise_status(a, MQA_STATUS_TIMEOUT);
            cf->abort = 1;
            return false;
        }
    }
}

// Waits (bounded, ignoring the abort flag) for in-flight work to land before
// the CTA exits.
__device__ __forceinline__ void wait_drain(uint64_t* bar, uint32_t parity, const KernelArgs& a) {
    const uint64_t t0 = ptx::globaltimer();
    while (!ptx::mbar_try_wait(bar, parity)) {
        if (ptx::globaltimer() - t0 > a.timeout_ns) {
            raise_status(a, MQA_STATUS_TIMEOUT);
            return;
        }
    }
}

// A bounded wait taken by lane 0 and broadcast, so the warp stays uniform.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile CtaFlags* cf,
                                          const KernelArgs& a, int lane) {
    bool ok = true;
    if (lane == 0) ok = wait_bounded(bar, parity, cf, a);
    return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
}

// Effective context length: negative counts as 0, values above ctx_cap are
// clamped (and flagged in validate mode), so no role can read past the block
// table or the output row.
__device__ __forceinline__ int clamp_ctx(const KernelArgs& a, int c) {
    if (c < 0) c = 0;
    if (c > a.ctx_cap) {
        if (a.flags & MQA_FLAG_VALIDATE) raise_status(a, MQA_STATUS_BAD_CONTEXT);
        c = a.ctx_cap;
    }
    return c;
}

__device__ __forceinline__ int units_of(int ctx) { return (ctx + kUnit - 1) / kUnit; }

// The context lengths of the rows a CTA touches, staged in shared memory at
// kernel start (rows past the cache fall back to global loads).
struct RowCache {
    const int32_t* ctx;  // shared memory
    int base, count;
    uint64_t* ready;     // completes when the cache has landed

    __device__ __forceinline__ int get(const KernelArgs& a, int b) const {
        const int i = b - base;
        return clamp_ctx(a, (i >= 0 && i < count) ? ctx[i] : __ldg(a.context_lens + b));
    }
};

__device__ __forceinline__ RowCache row_cache_view(const KernelArgs& a, int cta, const int32_t* src,
                                                   uint64_t* ready) {
    RowCache rc;
    rc.ctx = src;
    rc.ready = ready;
    rc.base = __ldg(a.schedule + 2 * cta);
    const int last = min(__ldg(a.schedule + 2 * cta + 2), a.batch - 1);
    rc.count = max(0, min(last - rc.base + 1, kRowCache));
    return rc;
}

// Issued by all 32 lanes of one warp: starts the copy of context_lens for the
// rows [first schedule row, last schedule row] of `cta` into `dst`, and makes
// `ready` (expected count 32) complete when the copies have landed.
__device__ __forceinline__ RowCache stage_rows(const KernelArgs& a, int cta, int32_t* dst,
                                               uint64_t* ready, int lane) {
    const RowCache rc = row_cache_view(a, cta, dst, ready);
    for (int i = lane; i < rc.count; i += 32) ptx::cp_async_4(dst + i, a.context_lens + rc.base + i);
    ptx::cp_async_mbar_arrive(ready);
    return rc;
}

// The work iterator. A CTA owns the schedule units from entry cta up to
// entry cta + 1; one unit (256 tokens of one row) is one pipeline stage and
// holds one or two 128-token MMA tiles (a tile that starts at or past the
// row's context does not exist). Rows without units are skipped. Every role
// (producer, MMA, epilogue, dequant) runs this same pure function of
// (schedule, context_lens), so all roles see the same sequence and the
// pipeline stays in step.
struct UnitIter {
    int b, j;          // row and unit within the row
    int end_b, end_j;
    int ctx;           // effective context of row b
    int idx;           // units visited so far
    int tiles;         // tiles visited so far (before this unit)
    int row_seq;       // rows with units visited so far, minus one (this unit's row)
    RowCache rows;

    __device__ __forceinline__ void init(const KernelArgs& a, int cta, const RowCache& rc) {
        rows = rc;
        b = __ldg(a.schedule + 2 * cta);
        j = __ldg(a.schedule + 2 * cta + 1);
        end_b = __ldg(a.schedule + 2 * cta + 2);
        end_j = __ldg(a.schedule + 2 * cta + 3);
        idx = 0;
        tiles = 0;
        row_seq = 0;
        if (b < 0) b = a.batch;  // corrupt schedule: no work
        if (j < 0) j = 0;
        ctx = (b < a.batch) ? rows.get(a, b) : 0;
        settle(a);
    }
    // Move forward to a real unit (or the end) from the current position.
    __device__ __forceinline__ void settle(const KernelArgs& a) {
        while (b < a.batch) {
            if (b == end_b && j == end_j) return;
            if (j < units_of(ctx)) return;
            ++b;
            j = 0;
            ctx = (b < a.batch) ? rows.get(a, b) : 0;
        }
    }
    __device__ __forceinline__ bool valid(const KernelArgs& a) const {
        return b < a.batch && !(b == end_b && j == end_j);
    }
    __device__ __forceinline__ int t0() const { return j * kUnit; }
    // MMA tiles in this unit: 2, or 1 if the context ends in its first half.
    __device__ __forceinline__ int ntiles() const { return (ctx - t0() > kTile) ? 2 : 1; }
    __device__ __forceinline__ void next(const KernelArgs& a) {
        ++idx;
        tiles += ntiles();
        ++j;
        const int b0 = b;
        settle(a);
        if (b != b0) ++row_seq;
    }
    // First unit of its row in this CTA (the CTA's first unit counts).
    __device__ __forceinline__ bool row_start(int first_j) const {
        return j == 0 || (idx == 0 && j == first_j);
    }
};

// Pages of one unit: npg loads of `rows` K rows each, starting at row
// `row_off` of the page named by block-table entry `pfirst` of the row.
struct UnitPages {
    int npg, rows, row_off, pfirst;
};

__device__ __forceinline__ UnitPages unit_pages(const UnitIter& it, const KernelArgs& a) {
    UnitPages up;
    const int t0 = it.t0();
    const int sh = a.ps_shift;
    if (sh >= 8) {  // page_size >= 256: one load of 256 rows
        up.npg = 1; up.rows = kUnit; up.row_off = t0 & ((1 << sh) - 1);
    } else {
        const int nv = min(kUnit, it.ctx - t0);
        up.npg = (nv + (1 << sh) - 1) >> sh; up.rows = 1 << sh; up.row_off = 0;
    }
    up.pfirst = t0 >> sh;
    return up;
}

// One producer warp (all 32 lanes, in lockstep); producer p of kProducers
// issues the units u with u % kProducers == p, so the per-unit work of
// kProducers warps overlaps. A producer waits only on the release of the
// stage it refills; since the MMA releases stages in unit order and a producer
// has already waited for the release of unit u - kProducers - NS before it
// reaches unit u, the parity of its wait cannot alias as long as
// NS >= kProducers (the launcher guarantees it).
// Block-table entries of the producer's next kPageLookahead units are fetched
// with cp.async into the producer's own ring (kPageLookahead + 1 units), entry
// k of a unit by lane k into that lane's own slot (so no cross-lane visibility
// is needed); per unit, lane 0 posts the expected bytes and lane k issues the
// loads of the unit's pages k, k + 32, ... Stages of the first ring round are
// known free and are not waited on.
// q and weights of every row are loaded by producer 0 alone, in row order
// (q buffer = row sequence number % 2): row R waits for the release of row
// R - 2, and is issued either before producer 0's first own unit at or past
// the row's first unit, or right after an own unit u when the row starts
// before u + kProducers. Row R - 2 then ends at or before a unit producer 0
// has issued (or one of the other producers, which never wait for producer
// 0, issues), so the wait cannot block the consumers it waits for.
//   q_load(q, b):                          loads into q buffer q, completing on qfull[q]
//   page_load(s, u, p, rows, row_off, pg): K rows (+ scales) of page p of unit u into stage s
//   row_bytes:                             bytes per token that complete on full[s]
//   q_bytes:                               bytes q_load makes arrive
template <class QLoad, class PageLoad>
__device__ __forceinline__ void producer_warp(const KernelArgs& a, int cta, const RowCache& rc,
                                              int p, int lane, uint64_t* full, uint64_t* empty,
                                              uint64_t* qfull, uint64_t* qempty, int32_t* pring,
                                              volatile CtaFlags* cf, uint32_t row_bytes,
                                              uint32_t q_bytes, QLoad q_load,
                                              PageLoad page_load) {
    constexpr int P = kProducers;
    constexpr int R = kPageLookahead + 1;  // page ring units per producer
    static_assert(P * R <= kPageRingUnits, "page ring too small");
    const int NS = a.num_stages;
    bool ok = warp_wait(rc.ready, 0, cf, a, lane);
    UnitIter it;
    it.init(a, cta, rc);
    const int first_j = it.j;
    UnitIter qit = it;   // producer 0: next unit whose row start is checked for a q load
    int q_last = -1;     // row sequence number of the last q load issued
    for (int i = 0; i < p && it.valid(a); ++i) it.next(a);
    int32_t* ring = pring + p * R * kMaxUnitPages;
    UnitIter fit = it;
    auto fetch_next = [&]() {  // block-table entries of this producer's next unit
        if (fit.valid(a)) {
            const UnitPages up = unit_pages(fit, a);
            for (int k = lane; k < up.npg; k += 32)
                ptx::cp_async_4(ring + ((fit.idx / P) % R) * kMaxUnitPages + k,
                                a.block_table + (int64_t)fit.b * a.max_pages + up.pfirst + k);
            for (int i = 0; i < P && fit.valid(a); ++i) fit.next(a);
        }
        ptx::cp_async_commit();
    };
    // producer 0: q loads of every row starting at or before unit umax
    auto q_upto = [&](int umax) -> bool {
        while (qit.valid(a) && qit.idx <= umax) {
            if (qit.row_start(first_j)) {
                const int q = qit.row_seq & 1;
                if (qit.row_seq >= 2 &&
                    !warp_wait(&qempty[q], ((qit.row_seq >> 1) & 1) ^ 1, cf, a, lane))
                    return false;
                if (lane == 0) {
                    ptx::mbar_arrive_expect_tx(&qfull[q], q_bytes);
                    q_load(q, qit.b);
                }
                q_last = qit.row_seq;
                __syncwarp();
            }
            qit.next(a);
        }
        return true;
    };
#pragma unroll 1
    for (int i = 0; i < kPageLookahead; ++i) fetch_next();

    // test only: with MQA_FLAG_TEST_DROP_ARRIVE, unit 1 is never filled
    const int dropped = (a.flags & MQA_FLAG_TEST_DROP_ARRIVE) != 0 ? 1 : -1;
    int last = -1;  // last unit issued by this producer
    while (ok && it.valid(a)) {
        const int u = it.idx;
        if (p == 0 && !q_upto(u)) break;
        const int s = u % NS;
        if (u >= NS && !warp_wait(&empty[s], ((uint32_t)(u / NS) & 1) ^ 1, cf, a, lane)) break;
        const UnitPages up = unit_pages(it, a);
        ptx::cp_async_wait<kPageLookahead - 1>();  // this unit's page indices landed
        if (u != dropped) {
            if (lane == 0)
                ptx::mbar_arrive_expect_tx(&full[s], (uint32_t)(up.npg * up.rows) * row_bytes);
            for (int k = lane; k < up.npg; k += 32) {
                int pg = ring[((u / P) % R) * kMaxUnitPages + k];
                if (pg < 0 || pg >= a.num_pages) {
                    if (a.flags & MQA_FLAG_VALIDATE) raise_status(a, MQA_STATUS_BAD_PAGE);
                    pg = 0;  // stay in bounds; the unit's values are then meaningless
                }
                page_load(s, u, k, up.rows, up.row_off, pg);
            }
        }
        last = u;
        if (lane == 0 && u < 16) MQA_TRACE_AT(40 + u);
        __syncwarp();
        fetch_next();
        if (p == 0 && !q_upto(u + P - 1)) { ok = false; break; }
        for (int i = 0; i < P && it.valid(a); ++i) it.next(a);
    }
    // producer 0: rows that start after its last own unit
    if (p == 0 && ok && !cf->abort) q_upto(0x7fffffff);
    ptx::cp_async_wait<0>();
    if (lane == 0) {
        if (p == 0) MQA_TRACE_AT(3);
        // On a normal finish the consumers have waited for every stage and q
        // buffer, so nothing is in flight. After an abort, wait (bounded) for
        // this producer's recent copies to land before the CTA exits.
        if (cf->abort) {
            for (int v = last; v >= 0 && v > last - NS; v -= P)
                if (v != dropped) wait_drain(&full[v % NS], (uint32_t)((v / NS) & 1), a);
            for (int r = q_last; r >= 0 && r > q_last - 2; --r)
                wait_drain(&qfull[r & 1], (uint32_t)((r >> 1) & 1), a);
        }
    }
    __syncwarp();
}

// Tail fill: -inf for every out[b][n][t] with t in [roundup(ctx_b, 128), L).
// Segments of 512 floats; segment (row r, k) belongs to CTA
// (r * nseg_max + k) mod num_ctas. One warp writes a segment with 16-byte
// stores; `warp` / `nwarps` split the rows among the calling warps.
__device__ __forceinline__ void tail_fill(const KernelArgs& a, int cta, int warp, int nwarps,
                                          int lane) {
    constexpr int kSeg = 512;
    constexpr int kBatch = 8;  // context loads in flight per lane
    const int L = a.out_len;
    const int nseg_max = (L + kSeg - 1) / kSeg;
    const int rows = a.batch * a.next_n;
    const float ni = __int_as_float(0xff800000);  // -inf
    const float4 ninf = make_float4(ni, ni, ni, ni);
    for (int r0 = warp * 32 * kBatch; r0 < rows; r0 += nwarps * 32 * kBatch) {
        int cv[kBatch];
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int r = r0 + u * 32 + lane;
            cv[u] = r < rows ? __ldg(a.context_lens + r / a.next_n) : 0;
        }
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int r = r0 + u * 32 + lane;
            int tstart = L, k0 = 0, nseg = 0;
            if (r < rows) {
                const int c = min(max(cv[u], 0), a.ctx_cap);
                tstart = min(L, ((c + kTile - 1) / kTile) * kTile);
                nseg = (L - tstart + kSeg - 1) / kSeg;
                const long long g = (long long)r * nseg_max;
                k0 = (int)(((long long)cta - g % a.num_ctas + a.num_ctas) % a.num_ctas);
            }
            uint32_t mine = __ballot_sync(0xffffffffu, r < rows && k0 < nseg);
            while (mine) {
                const int src = __ffs(mine) - 1;
                mine &= mine - 1;
                const int rr = r0 + u * 32 + src;
                const int ts = __shfl_sync(0xffffffffu, tstart, src);
                const int ns = __shfl_sync(0xffffffffu, nseg, src);
                int kk = __shfl_sync(0xffffffffu, k0, src);
                float* row = a.out + (long long)rr * L;
                for (; kk < ns; kk += a.num_ctas) {
                    const int s0 = ts + kk * kSeg;
                    const int s1 = min(L, s0 + kSeg);
                    for (int t = s0 + lane * 4; t < s1; t += 128)
                        *reinterpret_cast<float4*>(row + t) = ninf;
                }
            }
        }
    }
}

// Validate mode: does the schedule entry pair of `cta` match the current
// context_lens? (the reuse rule: a schedule stays valid only while every
// ceil(ctx_b / 256) is unchanged). One warp recomputes the unit prefix sums at
// this CTA's two entries and the total; a mismatch raises
// MQA_STATUS_STALE_SCHEDULE. The work itself is not changed.
__device__ __forceinline__ void check_schedule(const KernelArgs& a, int cta, int lane) {
    const int rs = __ldg(a.schedule + 2 * cta), js = __ldg(a.schedule + 2 * cta + 1);
    const int re = __ldg(a.schedule + 2 * cta + 2), je = __ldg(a.schedule + 2 * cta + 3);
    long long total = 0, before_s = 0, before_e = 0;
    int us = 0, ue = 0;
    for (int b = lane; b < a.batch; b += 32) {
        const int u = units_of(max(__ldg(a.context_lens + b), 0));
        total += u;
        if (b < rs) before_s += u;
        if (b < re) before_e += u;
        if (b == rs) us = u;
        if (b == re) ue = u;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        total += __shfl_xor_sync(0xffffffffu, total, o);
        before_s += __shfl_xor_sync(0xffffffffu, before_s, o);
        before_e += __shfl_xor_sync(0xffffffffu, before_e, o);
        us += __shfl_xor_sync(0xffffffffu, us, o);
        ue += __shfl_xor_sync(0xffffffffu, ue, o);
    }
    const long long S = a.num_ctas;
    auto expect = [&](long long i) { return i * (total / S) + min(i, total % S); };
    auto matches = [&](int r, int j, int u, long long before, long long want) {
        if (want >= total) return r == a.batch && j == 0;
        return r >= 0 && r < a.batch && j >= 0 && j < u && before + j == want;
    };
    const bool ok = matches(rs, js, us, before_s, expect(cta)) &&
                    matches(re, je, ue, before_e, expect(cta + 1));
    if (!ok && lane == 0) raise_status(a, MQA_STATUS_STALE_SCHEDULE);
}

}  // namespace mqa
