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
constexpr int kPageLookahead = 4;         // units whose block-table entries are fetched ahead
constexpr int kPageRingUnits = 8;         // units of block-table entries held (> kPageLookahead)
constexpr int kPageRing = kPageRingUnits * kMaxUnitPages;
constexpr int kMaxAccSlots = 8;           // TMEM accumulator slots (tiles in flight)

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
    L.scales = off;                               // stages x [256] fp32
    off += (uint32_t)stages * kUnit * 4;
    L.wbuf = off;                                 // 2 x [256] fp32 weights
    off += 2u * 256 * 4;
    L.rows = off;                                 // [kRowCache] context lengths
    off += kRowCache * 4;
    L.pages = off;                                // [kPageRing] block-table entries
    off += kPageRing * 4;
    L.bars = off;                                 // 2*stages + 6 + 2*kMaxAccSlots mbarriers
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
    RowCache rows;

    __device__ __forceinline__ void init(const KernelArgs& a, int cta, const RowCache& rc) {
        rows = rc;
        b = __ldg(a.schedule + 2 * cta);
        j = __ldg(a.schedule + 2 * cta + 1);
        end_b = __ldg(a.schedule + 2 * cta + 2);
        end_j = __ldg(a.schedule + 2 * cta + 3);
        idx = 0;
        tiles = 0;
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
        settle(a);
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

// The producer warp. Its two half-warps work in lockstep on alternate units
// (half g takes units g, g + 2, ...), so one pass of the loop issues two
// units. Block-table entries of the units kPageLookahead passes ahead are
// fetched with cp.async, entry p of a unit by lane p of its half into that
// lane's own slot of a shared ring (so no cross-lane visibility is needed);
// per unit, the half's leader posts the expected bytes and its lane p issues
// the loads of page p (pages p, p + 16, ... if a unit has more than 16).
// Stages of the first ring round are known free and are not waited on. Per
// row, the leader loads q and the weights; the two halves alternate q buffers
// only through the row order, which both follow.
//   q_load(q, b):                       loads into q buffer q, completing on qfull[q]
//   page_load(s, p, rows, row_off, pg): K rows + scales of page p into stage s
//   row_bytes:                          K + scale bytes per token
//   q_bytes:                            bytes q_load makes arrive
template <class QLoad, class PageLoad>
__device__ __forceinline__ void producer_warp(const KernelArgs& a, int cta, const RowCache& rc,
                                              int lane, uint64_t* full, uint64_t* empty,
                                              uint64_t* qfull, uint64_t* qempty, int32_t* pring,
                                              volatile CtaFlags* cf, uint32_t row_bytes,
                                              uint32_t q_bytes, QLoad q_load,
                                              PageLoad page_load) {
    const int NS = a.num_stages;
    const int half = lane >> 4;   // which alternate units this lane serves
    const int hl = lane & 15;     // lane within the half
    const bool ok0 = warp_wait(rc.ready, 0, cf, a, lane);
    // Both halves walk every unit; half g acts on units with idx % 2 == g.
    UnitIter it;
    it.init(a, cta, rc);
    UnitIter fit = it;
    int funit = 0;
    auto fetch_next = [&]() {  // fetch the next unit of this half
        if (fit.valid(a) && (fit.idx & 1) != half) fit.next(a);
        if (fit.valid(a)) {
            const UnitPages up = unit_pages(fit, a);
            for (int p = hl; p < up.npg; p += 16)
                ptx::cp_async_4(pring + (fit.idx % kPageRingUnits) * kMaxUnitPages + p,
                                a.block_table + (int64_t)fit.b * a.max_pages + up.pfirst + p);
            fit.next(a);
        }
        ++funit;
        ptx::cp_async_commit();
    };
#pragma unroll 1
    for (int i = 0; i < kPageLookahead; ++i) fetch_next();

    int prev_b = -1, qi = -1;
    // test only: with MQA_FLAG_TEST_DROP_ARRIVE, unit 1 is never filled
    const int dropped = (a.flags & MQA_FLAG_TEST_DROP_ARRIVE) != 0 ? 1 : -1;
    bool ok = ok0;
    while (ok && it.valid(a)) {
        // q for every new row, in row order (lane 0 alone; both halves step
        // through the same rows, so q buffers follow the MMA's order)
        if (it.b != prev_b) {
            ++qi;
            const int q = qi & 1;
            if (qi >= 2 && !warp_wait(&qempty[q], ((qi >> 1) & 1) ^ 1, cf, a, lane)) {
                --qi;
                break;
            }
            if (lane == 0) {
                ptx::mbar_arrive_expect_tx(&qfull[q], q_bytes);
                q_load(q, it.b);
            }
            prev_b = it.b;
        }
        // unit this half issues now: it.idx + half (if it exists)
        UnitIter mine = it;
        if (half == 1) mine.next(a);
        const bool have = mine.valid(a);
        // a second-half unit may start a new row: half 1 handles that row's q
        // next pass, when `it` reaches it; the MMA waits for q per row anyway
        const int u = mine.idx;
        const int s = u % NS;
        const uint32_t ph = (uint32_t)(u / NS) & 1;
        bool wok = true;
        if (have && u >= NS) {
            if (hl == 0) wok = wait_bounded(&empty[s], ph ^ 1, cf, a);
        }
        wok = __shfl_sync(0xffffffffu, wok ? 1 : 0, half * 16) != 0;
        if (!__all_sync(0xffffffffu, wok)) break;
        ptx::cp_async_wait<kPageLookahead - 1>();  // this half's unit page indices landed
        if (have) {
            const UnitPages up = unit_pages(mine, a);
            if (u != dropped) {
                if (hl == 0)
                    ptx::mbar_arrive_expect_tx(&full[s], (uint32_t)(up.npg * up.rows) * row_bytes);
                for (int p = hl; p < up.npg; p += 16) {
                    int pg = pring[(u % kPageRingUnits) * kMaxUnitPages + p];
                    if (pg < 0 || pg >= a.num_pages) {
                        if (a.flags & MQA_FLAG_VALIDATE) raise_status(a, MQA_STATUS_BAD_PAGE);
                        pg = 0;  // stay in bounds; the unit's values are then meaningless
                    }
                    page_load(s, p, up.rows, up.row_off, pg);
                }
            }
            if (hl == 0 && u < 16) MQA_TRACE_AT(40 + u);
        }
        __syncwarp();
        fetch_next();
        // advance both halves by two units; the row seen by half 1 this pass
        // must still get its q before the MMA needs it: handle it now
        if (it.valid(a)) it.next(a);
        if (it.valid(a) && it.b != prev_b) {
            ++qi;
            const int q = qi & 1;
            if (qi >= 2 && !warp_wait(&qempty[q], ((qi >> 1) & 1) ^ 1, cf, a, lane)) {
                --qi;
                break;
            }
            if (lane == 0) {
                ptx::mbar_arrive_expect_tx(&qfull[q], q_bytes);
                q_load(q, it.b);
            }
            prev_b = it.b;
        }
        if (it.valid(a)) it.next(a);
    }
    ptx::cp_async_wait<0>();
    if (lane == 0) {
        MQA_TRACE_AT(3);
        MQA_TRACE_VAL(10, it.idx);
        // Drain: wait (bounded) for every copy issued to land before exiting.
        const int n = it.idx;
        for (int i = max(0, n - NS); i < n; ++i)
            if (i != dropped) wait_drain(&full[i % NS], (uint32_t)((i / NS) & 1), a);
        for (int r = max(0, qi - 1); r <= qi; ++r)
            wait_drain(&qfull[r & 1], (uint32_t)((r >> 1) & 1), a);
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
