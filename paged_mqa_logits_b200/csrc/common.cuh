// Device-side pieces shared by the logits kernels: the argument block, the
// bounded pipeline wait and the work iterator that every warp role runs.
#pragma once
#include <cstdint>
#include "ptx.cuh"
#include "../../include/mqa_logits.h"

namespace mqa {

constexpr int kUnit = MQA_SCHEDULE_UNIT;  // tokens per schedule unit
constexpr int kTile = 128;                // tokens per MMA tile (M = 128)
constexpr int kTilesPerUnit = kUnit / kTile;
constexpr int kRowCache = 1024;  // context lengths of a CTA's rows staged in shared memory
constexpr int kPageRing = 256;   // block-table entries in flight (shared-memory ring)
constexpr int kPageLookahead = 8;  // tiles whose block-table entries are fetched ahead

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
    int32_t num_stages;       // K ring depth
    int32_t ctx_cap;          // min(out_len, max_pages * page_size)
    uint32_t flags;
    uint64_t timeout_ns;
};

// Shared-memory layout of the FP8 kernel: byte offsets from the 1024-aligned
// dynamic shared memory base. Used by the kernel and by the launcher.
struct Fp8Smem {
    uint32_t kst, qbuf, scales, wbuf, rows, pages, bars, misc, total;
};

__host__ __device__ inline int acc_stride(int npad) { return npad < 32 ? 32 : npad; }

__host__ __device__ inline Fp8Smem fp8_smem_layout(int D, int npad, int stages) {
    Fp8Smem L;
    uint32_t off = 0;
    L.kst = off;                                  // stages x [128 tokens][D] e4m3, swizzled
    off += (uint32_t)stages * kTile * D;
    L.qbuf = off;                                 // 2 x [npad][D] e4m3, swizzled
    off += 2u * npad * D;
    off = (off + 1023) & ~1023u;
    L.scales = off;                               // stages x [128] fp32
    off += (uint32_t)stages * kTile * 4;
    L.wbuf = off;                                 // 2 x [256] fp32 weights
    off += 2u * 256 * 4;
    L.rows = off;                                 // [kRowCache] context lengths
    off += kRowCache * 4;
    L.pages = off;                                // [kPageRing] block-table entries
    off += kPageRing * 4;
    L.bars = off;                                 // 2*stages + 10 mbarriers
    off += (uint32_t)(2 * stages + 10) * 8;
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
    L.kst = off;                                  // stages x [128 tokens][D/2] packed e2m1, swizzled
    off += (uint32_t)stages * kTile * (D / 2);
    off = (off + 1023) & ~1023u;
    L.qbuf = off;                                 // 2 x [D/64][npad][64] bf16 -> f16 in place
    off += 2u * npad * D * 2;
    L.scales = off;                               // stages x [128][D/16] e4m3 block scales
    off += (uint32_t)stages * kTile * (D / 16);
    off = (off + 15) & ~15u;
    L.wbuf = off;                                 // 2 x [256] fp32 weights
    off += 2u * 256 * 4;
    L.rows = off;                                 // [kRowCache] context lengths
    off += kRowCache * 4;
    L.pages = off;                                // [kPageRing] block-table entries
    off += kPageRing * 4;
    L.bars = off;                                 // 2*stages + 18 mbarriers
    off += (uint32_t)(2 * stages + 18) * 8;
    L.misc = off;                                 // TMEM address, abort flag, q maxima
    off += 48;
    L.total = off + 1024;
    return L;
}

// Shared across the CTA: set once any role gives up.
struct CtaFlags {
    int32_t abort;
};

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

// Effective context length of row b, read the same way by every role: values
// below 0 count as 0 and values above ctx_cap are clamped (and flagged in
// validate mode), so no role can read past the block table or the output row.
__device__ __forceinline__ int row_ctx(const KernelArgs& a, int b) {
    int c = __ldg(a.context_lens + b);
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

    __device__ __forceinline__ int get(const KernelArgs& a, int b) const {
        const int i = b - base;
        int c = (i >= 0 && i < count) ? ctx[i] : __ldg(a.context_lens + b);
        if (c < 0) c = 0;
        if (c > a.ctx_cap) {
            if (a.flags & MQA_FLAG_VALIDATE) raise_status(a, MQA_STATUS_BAD_CONTEXT);
            c = a.ctx_cap;
        }
        return c;
    }
};

// Issued by all 32 lanes of one warp: starts the copy of context_lens for the
// rows [first schedule row, last schedule row] of `cta` into `dst`, and makes
// `ready` (expected count 32) complete when the copies have landed.
__device__ __forceinline__ RowCache stage_rows(const KernelArgs& a, int cta, int32_t* dst,
                                               uint64_t* ready, int lane) {
    RowCache rc;
    rc.ctx = dst;
    rc.base = __ldg(a.schedule + 2 * cta);
    const int last = min(__ldg(a.schedule + 2 * cta + 2), a.batch - 1);
    rc.count = max(0, min(last - rc.base + 1, kRowCache));
    for (int i = lane; i < rc.count; i += 32) ptx::cp_async_4(dst + i, a.context_lens + rc.base + i);
    ptx::cp_async_mbar_arrive(ready);
    return rc;
}

// The same view of the cache for the roles that did not stage it.
__device__ __forceinline__ RowCache row_cache_view(const KernelArgs& a, int cta, const int32_t* src) {
    RowCache rc;
    rc.ctx = src;
    rc.base = __ldg(a.schedule + 2 * cta);
    const int last = min(__ldg(a.schedule + 2 * cta + 2), a.batch - 1);
    rc.count = max(0, min(last - rc.base + 1, kRowCache));
    return rc;
}

// The work iterator. A CTA owns the schedule units from entry cta up to
// entry cta + 1; each unit is split into 128-token tiles, and a tile that
// starts at or past the row's context is not a tile at all. Rows without
// units are skipped. Every role (producer, MMA, epilogue) runs this same pure
// function of (schedule, context_lens), so all roles see the same tile
// sequence and the pipeline stays in step.
struct TileIter {
    int b, j, k;       // row, unit within the row, tile within the unit
    int end_b, end_j;
    int ctx;           // effective context of row b
    int idx;           // tiles visited so far
    RowCache rows;

    __device__ __forceinline__ void init(const KernelArgs& a, int cta, const RowCache& rc) {
        rows = rc;
        b = __ldg(a.schedule + 2 * cta);
        j = __ldg(a.schedule + 2 * cta + 1);
        end_b = __ldg(a.schedule + 2 * cta + 2);
        end_j = __ldg(a.schedule + 2 * cta + 3);
        k = 0;
        idx = 0;
        if (b < 0) b = a.batch;  // corrupt schedule: no work
        if (j < 0) j = 0;
        ctx = (b < a.batch) ? rows.get(a, b) : 0;
        settle(a);
    }
    // Move forward to a real tile (or the end) from the current position.
    __device__ __forceinline__ void settle(const KernelArgs& a) {
        while (b < a.batch) {
            if (b == end_b && j == end_j && k == 0) return;
            if (j < units_of(ctx) && (j * kUnit + k * kTile) < ctx) return;
            // past the row's last tile: next row with context
            ++b;
            j = 0;
            k = 0;
            ctx = (b < a.batch) ? rows.get(a, b) : 0;
        }
    }
    __device__ __forceinline__ bool valid(const KernelArgs& a) const {
        return b < a.batch && !(b == end_b && j == end_j && k == 0);
    }
    __device__ __forceinline__ void next(const KernelArgs& a) {
        ++idx;
        if (++k == kTilesPerUnit || (j * kUnit + k * kTile) >= ctx) {
            k = 0;
            ++j;
        }
        settle(a);
    }
    __device__ __forceinline__ int t0() const { return j * kUnit + k * kTile; }
};

// Pages of one tile: npg loads of `rows` K rows each, starting at row
// `row_off` of the page named by block-table entry `pfirst` of the row.
struct TilePages {
    int npg, rows, row_off, pfirst;
};

__device__ __forceinline__ TilePages tile_pages(const TileIter& it, int ps) {
    TilePages tp;
    const int t0 = it.t0();
    if (ps >= kTile) {
        tp.npg = 1; tp.rows = kTile; tp.row_off = t0 % ps;
    } else {
        const int nv = min(kTile, it.ctx - t0);
        tp.npg = (nv + ps - 1) / ps; tp.rows = ps; tp.row_off = 0;
    }
    tp.pfirst = t0 / ps;
    return tp;
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
