// Device-side pieces shared by the logits kernels: the argument block, shared
// memory layouts, the bounded pipeline wait, the per-CTA work table (built once
// per chunk by one warp, walked by every role), the producer warp, the -inf
// tail fill and the validate-mode schedule check.
#pragma once
#include <cstdint>
#include "ptx.cuh"
#define MQA_LOGITS_TEST_HOOKS
#include "mqa_logits.h"

namespace mqa {

constexpr int kUnit = MQA_SCHEDULE_UNIT;  // tokens per schedule unit = one pipeline stage
constexpr int kTile = 128;                // tokens per MMA tile (M = 128)
constexpr int kProducers = 3;             // producer warps; warp p issues units p, p + 3, ...
constexpr int kChunk = 32;                // work-table units per chunk (at most): one builder pass
constexpr int kChunkPages = 512;          // block-table entries per chunk
constexpr int kTableUsers = 16;           // warps that walk the table (all kernels)
constexpr int kMaxAccSlots = 8;           // TMEM accumulator slots (tiles in flight)

// Everything a logits kernel needs besides its tensor maps (by value).
struct KernelArgs {
    const uint8_t* kv;
    const uint8_t* q;         // q, for the L2 warm-up only (the kernels read it through tm_q)
    int64_t q_bytes;
    const int32_t* block_table;
    const int32_t* context_lens;
    const float* weights;
    const int32_t* schedule;
    float* out;
    int32_t* status;          // the caller's optional status word (may be NULL)
    uint32_t* lib_status;     // the library's own word on this device (never NULL)
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

// One unit of a CTA's work: 256 tokens [t0, t0 + 256) of row b (context ctx),
// whose first MMA tile is the CTA's tile number `tile`.
struct UnitDesc {
    int32_t b, t0, ctx, tile;
};

// Work table in shared memory: two chunk buffers, each with up to kChunk unit
// descriptors, per unit its row sequence number * 2 + (first unit of its row
// in this CTA), and the unit's block-table entries; plus the chunk's unit
// count. 16-byte aligned.
constexpr uint32_t kTableBytes = 2u * (kChunk * 16 + kChunk * 4 + kChunkPages * 4) + 16;

// Shared-memory layout of the FP8 kernel: byte offsets from the 1024-aligned
// dynamic shared memory base. Used by the kernel and by the launcher.
struct Fp8Smem {
    uint32_t kst, qbuf, wbuf, table, bars, misc, total;
};

constexpr int kFp8Bars = 9 + 2 * kMaxAccSlots;  // + 2 per stage

__host__ __device__ inline Fp8Smem fp8_smem_layout(int D, int npad, int stages) {
    Fp8Smem L;
    uint32_t off = 0;
    L.kst = off;                                  // stages x [256 tokens][D] e4m3, swizzled
    off += (uint32_t)stages * kUnit * D;
    L.qbuf = off;                                 // 2 x [npad][D] e4m3, swizzled
    off += 2u * npad * D;
    off = (off + 15) & ~15u;
    L.wbuf = off;                                 // 2 x [256] fp32 weights
    off += 2u * 256 * 4;
    L.table = off;                                // work table
    off += kTableBytes;
    L.bars = off;                                 // 2*stages + kFp8Bars mbarriers
    off += (uint32_t)(2 * stages + kFp8Bars) * 8;
    L.misc = off;                                 // TMEM address, CtaFlags
    off += 32;
    L.total = off + 1024;                         // slack for aligning the base
    return L;
}

// Shared-memory layout of the FP4 kernel. A K page (ps tokens: ps x D/2 packed
// e2m1 bytes, then ps x D/16 e4m3 scale bytes, 9 ps D / 16 bytes in all) comes
// in whole with one tensor copy, viewed as 9 ps / 16 rows of D bytes (two
// tokens' codes a row) with the D-byte swizzle (128 B for D = 128, 64 B for
// D = 64); each page gets its own slot, aligned to the swizzle atom so the
// pattern is a function of the offset within the slot.
struct Fp4Smem {
    uint32_t kst, page_slot, stage, qbuf, wbuf, table, bars, misc, total;
};

constexpr int kFp4Bars = 13 + 4 * kMaxAccSlots;  // + 2 per stage

__host__ __device__ inline uint32_t fp4_page_slot(int D, int page_size) {
    const uint32_t bytes = (uint32_t)(9 * page_size * D / 16);
    const uint32_t atom = D >= 128 ? 1024u : 512u;
    return (bytes + atom - 1) / atom * atom;
}

__host__ __device__ inline Fp4Smem fp4_smem_layout(int D, int npad, int stages, int page_size) {
    Fp4Smem L;
    uint32_t off = 0;
    const int pages = page_size >= kUnit ? 1 : kUnit / page_size;
    L.page_slot = fp4_page_slot(D, page_size);
    L.stage = (uint32_t)pages * L.page_slot;
    L.kst = off;                                  // stages x pages x [page slot]
    off += (uint32_t)stages * L.stage;
    off = (off + 1023) & ~1023u;
    L.qbuf = off;                                 // 2 x [D/64][npad][64] bf16 -> f16 in place
    off += 2u * npad * D * 2;
    L.wbuf = off;                                 // 2 x [256] fp32 weights
    off += 2u * 256 * 4;
    L.table = off;                                // work table
    off += kTableBytes;
    L.bars = off;                                 // 2*stages + kFp4Bars mbarriers
    off += (uint32_t)(2 * stages + kFp4Bars) * 8;
    L.misc = off;                                 // TMEM address, CtaFlags, q maxima, q exponents
    off += 64;
    L.total = off + 1024;
    return L;
}

// Shared-memory layout of the block-scaled FP4 kernel (q and K both e2m1 with
// e4m3 scales per 16 elements).
struct Nvfp4Smem {
    uint32_t kst, qbuf, ksf, qsf, kraw, qraw, wbuf, table, bars, misc, total;
};

constexpr int kNvfp4Bars = 9 + 2 * kMaxAccSlots;  // + 2 per stage

__host__ __device__ inline Nvfp4Smem nvfp4_smem_layout(int D, int npad, int stages) {
    const int rb = D / 2, sb = D / 16, ks = D / 64;
    Nvfp4Smem L;
    uint32_t off = 0;
    L.kst = off;                                  // stages x [256 tokens][D/2] packed e2m1, swizzled
    off += (uint32_t)stages * kUnit * rb;
    off = (off + 1023) & ~1023u;
    L.qbuf = off;                                 // 2 x [npad][D/2] packed e2m1, swizzled
    off += 2u * npad * rb;
    off = (off + 1023) & ~1023u;
    L.ksf = off;                                  // stages x 2 tiles x D/64 scale blocks of 512 B
    off += (uint32_t)stages * 2 * ks * 512;
    L.qsf = off;                                  // 2 x D/64 scale blocks of 512 B
    off += 2u * ks * 512;
    L.kraw = off;                                 // stages x [256][D/16] e4m3 scales as loaded
    off += (uint32_t)stages * kUnit * sb;
    L.qraw = off;                                 // 2 x [128][D/16] e4m3 scales as loaded
    off += 2u * 128 * sb;
    off = (off + 15) & ~15u;
    L.wbuf = off;                                 // 2 x [256] fp32 weights
    off += 2u * 256 * 4;
    L.table = off;                                // work table
    off += kTableBytes;
    L.bars = off;                                 // 2*stages + kNvfp4Bars mbarriers
    off += (uint32_t)(2 * stages + kNvfp4Bars) * 8;
    L.misc = off;                                 // TMEM address, CtaFlags
    off += 32;
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
int launch_nvfp4_logits(int H, int D, const LaunchSpec& ls, const CUtensorMap& tm_k,
                        const CUtensorMap& tm_q, const KernelArgs& args);

// Shared across the CTA: `abort` is set once any role gives up; `consumed`
// counts the units whose stage the consumer has seen full (so a unit below it
// has no copies in flight); `q_seen` counts the rows whose q buffer a consumer
// has seen full.
struct CtaFlags {
    int32_t abort;
    int32_t consumed;
    int32_t q_seen;
};
#ifdef MQA_DEBUG

// Debug builds: per-CTA counts that the roles leave for the exit checks (-1
// until written): the MMA walker's units, tiles, rows and table chunks, the
// builder's placed units, each producer's and each epilogue warp's walked
// units, and each epilogue warp's tiles.
enum : int {
    kDbgUnits = 0, kDbgTiles = 1, kDbgRows = 2, kDbgChunks = 3, kDbgBuilt = 4,
    kDbgProd = 5,        // + producer index (up to 3)
    kDbgEpiUnits = 8,    // + epilogue warp (up to 16)
    kDbgEpiTiles = 24,   // + epilogue warp (up to 16)
    kDbgSlots = 40
};
__shared__ int32_t g_mqa_dbg[kDbgSlots];
#endif

// Issued before the grid-dependency wait, by the warps that are idle at that
// point (thread t of nt per CTA): L2 prefetches of the block table, the
// context lengths, q and the weights, spread over all CTAs, and one line per
// 2 MiB of the KV cache so its address translations are cached before the
// gather starts. Prefetches are hints that return no data, and L2 is the
// point of coherence, so this is safe even while the previous kernel in the
// stream is still writing these inputs.
__device__ __forceinline__ void warm_inputs(const KernelArgs& a, int cta, int t, int nt) {
    const int64_t stride = (int64_t)a.num_ctas * nt;
    const int64_t first = (int64_t)cta * nt + t;
    auto lines = [&](const void* base, int64_t bytes) {
        const uint8_t* p = static_cast<const uint8_t*>(base);
        for (int64_t l = first; l * 128 < bytes; l += stride) ptx::prefetch_l2(p + l * 128);
    };
    lines(a.block_table, (int64_t)a.batch * a.max_pages * 4);
    lines(a.context_lens, (int64_t)a.batch * 4);
    lines(a.weights, (int64_t)a.batch * a.hn * 4);
    lines(a.q, a.q_bytes);
    const int64_t kv_bytes = (int64_t)a.num_pages * a.page_bytes;
    for (int64_t l = first; (l << 21) < kv_bytes; l += stride) ptx::prefetch_l2(a.kv + (l << 21));
}

__device__ __forceinline__ void raise_status(const KernelArgs& a, uint32_t bits) {
    atomicOr(a.lib_status, bits);
    if (a.status != nullptr) atomicOr(reinterpret_cast<uint32_t*>(a.status), bits);
}

// Hardware suspension per wait attempt: long enough that a waiting warp is
// parked rather than polling, short enough that the abort flag and the timeout
// are still checked often.
constexpr uint32_t kWaitSliceNs = 20000;

// Waits for phase `parity` of `bar` to complete. Returns false if the CTA was
// aborted by another role or if the wait exceeded the timeout (then the
// status word gets MQA_STATUS_TIMEOUT and the CTA is aborted). Never traps.
__device__ __forceinline__ bool wait_bounded(uint64_t* bar, uint32_t parity,
                                             volatile CtaFlags* cf, const KernelArgs& a) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = ptx::globaltimer();
    while (true) {
        if (ptx::mbar_try_wait_sleep(bar, parity, kWaitSliceNs)) return true;
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
    while (!ptx::mbar_try_wait_sleep(bar, parity, kWaitSliceNs)) {
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
// clamped (both flagged in validate mode), so no role can read past the block
// table or the output row.
__device__ __forceinline__ int clamp_ctx(const KernelArgs& a, int c) {
    if (c < 0 || c > a.ctx_cap) {
        if (a.flags & MQA_FLAG_VALIDATE) raise_status(a, MQA_STATUS_BAD_CONTEXT);
        c = c < 0 ? 0 : a.ctx_cap;
    }
    return c;
}

__device__ __forceinline__ int units_of(int ctx) { return (ctx + kUnit - 1) / kUnit; }

// Device view of the work table (see kTableBytes). The builder warp fills
// chunk k into buffer k % 2 after every table user released chunk k - 2; a
// chunk with fewer than `cap` units is the last one.
struct Table {
    UnitDesc* desc;    // [2][kChunk]
    int32_t* info;     // [2][kChunk]: row sequence number * 2 + row start
    int32_t* pages;    // [2][kChunkPages]: unit i's entries at i * upp
    int32_t* count;    // [2]
    uint64_t* full;    // [2]: the builder's 32 lanes arrive
    uint64_t* empty;   // [2]: kTableUsers warps arrive
    int cap;           // units per chunk: min(kChunk, kChunkPages / upp)
    int upp;           // block-table entries per unit (256 / page_size, at least 1)
};

__device__ __forceinline__ Table table_view(uint8_t* p, uint64_t* bars, const KernelArgs& a) {
    Table T;
    T.desc = reinterpret_cast<UnitDesc*>(p);
    T.info = reinterpret_cast<int32_t*>(p + 2 * kChunk * 16);
    T.pages = T.info + 2 * kChunk;
    T.count = T.pages + 2 * kChunkPages;
    T.full = bars;
    T.empty = bars + 2;
    T.upp = a.ps_shift >= 8 ? 1 : (kUnit >> a.ps_shift);
    T.cap = min(kChunk, kChunkPages / T.upp);
    return T;
}

// Walks the table one unit at a time. kWarp: the whole warp calls next() in
// lockstep (lane 0 waits and releases); otherwise one thread does.
struct TableCursor {
    int k = -1, i = 0, n = 0;

    // 0: at a unit; 1: no more units; 2: the CTA was aborted.
    template <bool kWarp>
    __device__ __forceinline__ int next(const Table& T, volatile CtaFlags* cf, const KernelArgs& a,
                                        int lane) {
        if (k >= 0) {
            if (++i < n) return 0;
            release<kWarp>(T, lane);
            if (n < T.cap) return 1;
        }
        ++k;
        i = 0;
        const uint32_t par = (uint32_t)(k >> 1) & 1;
        const bool ok = kWarp ? warp_wait(&T.full[k & 1], par, cf, a, lane)
                              : wait_bounded(&T.full[k & 1], par, cf, a);
        if (!ok) return 2;
        n = T.count[k & 1];
        if (n == 0) {
            release<kWarp>(T, lane);
            return 1;
        }
        return 0;
    }
    template <bool kWarp>
    __device__ __forceinline__ void release(const Table& T, int lane) const {
        if (kWarp) __syncwarp();
        if (!kWarp || lane == 0) ptx::mbar_arrive(&T.empty[k & 1]);
    }
    __device__ __forceinline__ int unit(const Table& T) const { return k * T.cap + i; }
    __device__ __forceinline__ UnitDesc desc(const Table& T) const {
        return T.desc[(k & 1) * kChunk + i];
    }
    __device__ __forceinline__ int info(const Table& T) const {
        return T.info[(k & 1) * kChunk + i];
    }
    __device__ __forceinline__ const int32_t* pages(const Table& T) const {
        return T.pages + (k & 1) * kChunkPages + i * T.upp;
    }
};

// MMA tiles in a unit: 2, or 1 when the row's context ends in its first half.
__device__ __forceinline__ int unit_tiles(const UnitDesc& d) { return d.ctx - d.t0 > kTile ? 2 : 1; }

// Block-table entries a unit needs: npg page loads of `rows` K rows each,
// starting at row `row_off` of each page; the first entry is t0 / page_size.
__device__ __forceinline__ void unit_loads(const UnitDesc& d, int sh, int& npg, int& rows,
                                           int& row_off) {
    if (sh >= 8) {  // page_size >= 256: one load of 256 rows
        npg = 1; rows = kUnit; row_off = d.t0 & ((1 << sh) - 1);
    } else {
        npg = (min(kUnit, d.ctx - d.t0) + (1 << sh) - 1) >> sh; rows = 1 << sh; row_off = 0;
    }
}

// The builder warp (all 32 lanes). A CTA owns the schedule units from entry
// cta up to entry cta + 1, in row order; one unit (256 tokens of one row) is
// one pipeline stage with one or two 128-token MMA tiles. Rows are taken 32 at
// a time, one per lane: its effective context, the units it contributes
// (respecting the first and the end position), warp prefix sums of units and
// tiles and a ballot of new rows place every unit in the chunk; lane q then
// writes units q, q + 32, ... (finding its row by a shuffle binary search over
// the prefix sums) with the unit's block-table entries. To shorten the start,
// the builder itself issues the loads of the first `first` units (the first
// ring round, whose stages are free) and the q loads of the first two rows
// (whose q buffers are free); the producers take over from there.
template <class QLoad, class PageLoad>
__device__ __forceinline__ void build_table(const KernelArgs& a, int cta, const Table& T,
                                            volatile CtaFlags* cf, int lane, int first,
                                            uint64_t* full, uint64_t* qfull, uint32_t row_bytes,
                                            uint32_t q_bytes, QLoad q_load, PageLoad page_load) {
    constexpr unsigned kAll = 0xffffffffu;
    int cb = ptx::ld_cg(a.schedule + 2 * cta), cj = ptx::ld_cg(a.schedule + 2 * cta + 1);
    const int eb = ptx::ld_cg(a.schedule + 2 * cta + 2), ej = ptx::ld_cg(a.schedule + 2 * cta + 3);
    if (cb < 0) cb = a.batch;  // corrupt schedule: no work
    if (cj < 0) cj = 0;
    const int last = min(eb, a.batch - 1);
    const int sh = a.ps_shift;
    // test only: with MQA_FLAG_TEST_DROP_ARRIVE, unit 1 is never filled
    const int dropped = (a.flags & MQA_FLAG_TEST_DROP_ARRIVE) != 0 ? 1 : -1;
    int tiles = 0, rows_seen = 0, last_row = -1, issued = 0;
    // After an abort, wait (bounded) for the copies this warp issued itself
    // and no consumer has seen yet (their barriers are still in their first
    // phase: a stage or q buffer is refilled only after it was consumed), so
    // the CTA never exits with them in flight.
    auto drain_own = [&]() {
        if (cf->abort && lane == 0) {
            for (int u = max(cf->consumed, 0); u < issued; ++u)
                if (u != dropped) wait_drain(&full[u], 0, a);
            for (int r = max(cf->q_seen, 0); r < min(rows_seen, 2); ++r)
                wait_drain(&qfull[r], 0, a);
        }
        __syncwarp();
    };
    for (int k = 0;; ++k) {
        const int buf = k & 1;
        if (k >= 2 && !warp_wait(&T.empty[buf], (uint32_t)((k - 2) >> 1) & 1, cf, a, lane)) {
            drain_own();
            return;
        }
        UnitDesc* D = T.desc + buf * kChunk;
        int32_t* I = T.info + buf * kChunk;
        int32_t* PG = T.pages + buf * kChunkPages;
        int filled = 0;
        while (filled < T.cap && cb <= last) {
            const int r = cb + lane;
            const bool in = r <= last;
            const int c = in ? clamp_ctx(a, ptx::ld_cg(a.context_lens + r)) : 0;
            const int jb = lane == 0 ? cj : 0;
            const int nu = units_of(c);
            const int je = r == eb ? min(nu, ej) : nu;
            const int n = in ? max(je - jb, 0) : 0;
            int incl = n;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int v = __shfl_up_sync(kAll, incl, o);
                if (lane >= o) incl += v;
            }
            const int excl = incl - n;
            const int take = min(__shfl_sync(kAll, incl, 31), T.cap - filled);
            const int got = max(0, min(incl, take) - excl);  // this row's units placed now
            // only a row's final unit can have one tile
            const bool ends = got > 0 && jb + got == nu && c - ((nu - 1) << 8) <= kTile;
            const int nt = 2 * got - (ends ? 1 : 0);
            int tincl = nt;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int v = __shfl_up_sync(kAll, tincl, o);
                if (lane >= o) tincl += v;
            }
            const int tbase = tiles + tincl - nt;
            const bool newrow = got > 0 && r != last_row;
            const unsigned nr = __ballot_sync(kAll, newrow);
            const int rseq = newrow ? rows_seen + __popc(nr & ((1u << lane) - 1)) : rows_seen - 1;
            // the first two rows' q buffers are free: load them now
            if (newrow && rseq < 2) {
                ptx::mbar_arrive_expect_tx(&qfull[rseq], q_bytes);
                q_load(rseq, r);
            }
            for (int q0 = 0; q0 < take; q0 += 32) {
                const int q = q0 + lane;
                int src = 0;  // the lane whose row holds unit q: first lane with incl > q
#pragma unroll
                for (int st = 16; st > 0; st >>= 1) {
                    const int v = __shfl_sync(kAll, incl, src + st - 1);
                    if (v <= q) src += st;
                }
                const int s_jb = __shfl_sync(kAll, jb, src);
                const int s_excl = __shfl_sync(kAll, excl, src);
                const int s_c = __shfl_sync(kAll, c, src);
                const int s_tb = __shfl_sync(kAll, tbase, src);
                const int s_seq = __shfl_sync(kAll, rseq, src);
                const bool s_new = __shfl_sync(kAll, newrow ? 1 : 0, src) != 0;
                if (q < take) {
                    const int jj = q - s_excl;
                    const int row = cb + src;
                    const int u = k * T.cap + filled + q;  // CTA-local unit index
                    UnitDesc d;
                    d.b = row;
                    d.t0 = (s_jb + jj) << 8;
                    d.ctx = s_c;
                    d.tile = s_tb + 2 * jj;
                    D[filled + q] = d;
                    I[filled + q] = s_seq * 2 + ((s_new && jj == 0) ? 1 : 0);
                    int npg, rows, row_off;
                    unit_loads(d, sh, npg, rows, row_off);
                    const int32_t* src_bt = a.block_table + (int64_t)row * a.max_pages + (d.t0 >> sh);
                    int32_t* dst = PG + (filled + q) * T.upp;
                    const bool issue = u < first && u != dropped;
                    if (issue)
                        ptx::mbar_arrive_expect_tx(&full[u], (uint32_t)(npg * rows) * row_bytes);
                    for (int x0 = 0; x0 < npg; x0 += 4) {  // four entries in flight at a time
                        int pgv[4];
#pragma unroll
                        for (int i = 0; i < 4; ++i) pgv[i] = x0 + i < npg ? ptx::ld_cg(src_bt + x0 + i) : 0;
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            if (x0 + i >= npg) break;
                            int pg = pgv[i];
                            dst[x0 + i] = pg;
                            if (issue) {
                                if (pg < 0 || pg >= a.num_pages) {
                                    if (a.flags & MQA_FLAG_VALIDATE) raise_status(a, MQA_STATUS_BAD_PAGE);
                                    pg = 0;  // stay in bounds; the unit's values are then meaningless
                                }
                                page_load(u, u, x0 + i, rows, row_off, pg);
                            }
                        }
                    }
                }
            }
            // advance past the placed units (all uniform)
            tiles += __shfl_sync(kAll, tincl, 31);
            rows_seen += __popc(nr);
            if (take > 0) {
                const int lr = __popc(__ballot_sync(kAll, incl < take));  // lane of unit take - 1
                last_row = cb + lr;
            }
            if (take == __shfl_sync(kAll, incl, 31)) {
                cb += 32;
                cj = 0;
            } else {
                const int nl = __popc(__ballot_sync(kAll, incl <= take));  // lane of unit `take`
                cj = __shfl_sync(kAll, jb, nl) + (take - __shfl_sync(kAll, excl, nl));
                cb += nl;
            }
            filled += take;
            issued = min(first, k * T.cap + filled);
        }
        if (lane == 0) T.count[buf] = filled;
        ptx::mbar_arrive(&T.full[buf]);  // releases this lane's table writes
        if (filled < T.cap) {
#ifdef MQA_DEBUG
            if (lane == 0) g_mqa_dbg[kDbgBuilt] = k * T.cap + filled;
#endif
            drain_own();
            return;
        }
    }
}

// Units the builder loads itself (see build_table): at most `want`, within the
// ring and the first chunk; the producers start after.
__device__ __forceinline__ int builder_units(const KernelArgs& a, const Table& T, int want) {
    return min(min(a.num_stages, want), T.cap);
}

// One producer warp (all 32 lanes, in lockstep); producer p of NP issues the
// units u with u % NP == p, so the per-unit work of NP warps overlaps (NP = 1:
// one warp issues every unit, in unit order). A producer waits only on the
// release of the stage it refills; since the MMA releases stages in unit order
// and a producer has already waited for the release of unit u - NP - NS before
// it reaches unit u, the parity of its wait cannot alias as long as NS >= NP
// (the launcher guarantees it). Per unit, lane 0 posts the expected bytes and
// lane k issues the loads of the unit's pages k, k + 32, ... (block-table
// entries come from the work table). Units below `first` were issued by the
// builder warp.
// q and weights of every row from the third on are loaded by producer 0,
// which walks every unit in order and loads q at each row start (q buffer =
// row sequence number % 2) after the release of row R - 2. That row ends at or
// before unit u - 2, and every unit before u is issued by producer 0 already
// or by the other producers, which never wait for producer 0, so the wait
// cannot block the consumers it waits for.
//   q_load(q, b):                          loads into q buffer q, completing on qfull[q]
//   page_load(s, u, p, rows, row_off, pg): K rows (+ scales) of page p of unit u into stage s
//   row_bytes:                             bytes per token that complete on full[s]
//   q_bytes:                               bytes q_load makes arrive
template <int NP, class QLoad, class PageLoad>
__device__ __forceinline__ void producer_warp(const KernelArgs& a, const Table& T, int p, int lane,
                                              int first,
                                              uint64_t* full, uint64_t* empty, uint64_t* qfull,
                                              uint64_t* qempty, volatile CtaFlags* cf,
                                              uint32_t row_bytes, uint32_t q_bytes, QLoad q_load,
                                              PageLoad page_load) {
    const int NS = a.num_stages;
    const int sh = a.ps_shift;
    // test only: with MQA_FLAG_TEST_DROP_ARRIVE, unit 1 is never filled
    const int dropped = (a.flags & MQA_FLAG_TEST_DROP_ARRIVE) != 0 ? 1 : -1;
    int last = -1;    // last unit issued by this producer
    int q_last = -1;  // row sequence number of the last q load issued
    // stage and phase of this producer's next unit u: s = u % NS, ph = (u / NS) & 1,
    // advanced by NP units at a time (no division on the issue path)
    int s = p, ph = 0;
    TableCursor cur;
    int rc;
#ifdef MQA_DEBUG
    int walked = 0;
#endif
    while ((rc = cur.next<true>(T, cf, a, lane)) == 0) {
        const int u = cur.unit(T);
#ifdef MQA_DEBUG
        ++walked;
#endif
        if (p == 0) {
            const int info = cur.info(T);
            if (info & 1) {
                const int rs = info >> 1, q = rs & 1;
                q_last = rs;
                if (rs >= 2) {  // rows 0 and 1 were loaded by the builder
                    if (!warp_wait(&qempty[q], ((uint32_t)(rs >> 1) & 1) ^ 1, cf, a, lane)) {
                        rc = 2;
                        break;
                    }
                    if (lane == 0) {
                        ptx::mbar_arrive_expect_tx(&qfull[q], q_bytes);
                        q_load(q, cur.desc(T).b);
                    }
                    __syncwarp();
                }
            }
        }
        if (u % NP != p) continue;
        const int us = s;
        const uint32_t uph = (uint32_t)ph;
        s += NP;  // NS >= NP: wraps at most once
        if (s >= NS) { s -= NS; ph ^= 1; }
        if (u < first) {  // issued by the builder; counted here for the abort drain
            last = u;
            continue;
        }
        if (u >= NS && !warp_wait(&empty[us], uph ^ 1, cf, a, lane)) {
            rc = 2;
            break;
        }
        if (u != dropped) {
            const UnitDesc d = cur.desc(T);
            int npg, rows, row_off;
            unit_loads(d, sh, npg, rows, row_off);
            if (lane == 0)
                ptx::mbar_arrive_expect_tx(&full[us], (uint32_t)(npg * rows) * row_bytes);
            const int32_t* pgs = cur.pages(T);
            for (int k = lane; k < npg; k += 32) {
                int pg = pgs[k];
                if (pg < 0 || pg >= a.num_pages) {
                    if (a.flags & MQA_FLAG_VALIDATE) raise_status(a, MQA_STATUS_BAD_PAGE);
                    pg = 0;  // stay in bounds; the unit's values are then meaningless
                }
                page_load(us, u, k, rows, row_off, pg);
            }
        }
        last = u;
        __syncwarp();
    }
#ifdef MQA_DEBUG
    if (rc == 1 && lane == 0) g_mqa_dbg[kDbgProd + p] = walked;
#endif
    if (lane == 0) {
        // On a normal finish the consumers have waited for every stage and q
        // buffer, so nothing is in flight. After an abort, wait (bounded) for
        // this producer's recent copies to land before the CTA exits.
        if (cf->abort) {
            // units at or past `consumed` were not refilled, so their parity
            // cannot alias
            const int done = cf->consumed;
            for (int v = last; v >= done && v > last - NS; v -= NP)
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
    constexpr int kBatch = 4;  // context loads in flight per lane
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
            cv[u] = r < rows ? ptx::ld_cg(a.context_lens + r / a.next_n) : 0;
        }
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int r = r0 + u * 32 + lane;
            int tstart = L, k0 = 0, nseg = 0;
            if (r < rows) {
                const int c = min(max(cv[u], 0), a.ctx_cap);
                tstart = min(L, ((c + kTile - 1) / kTile) * kTile);
                nseg = (L - tstart + kSeg - 1) / kSeg;
                // (r * nseg_max) mod S without 64-bit arithmetic
                const unsigned S = (unsigned)a.num_ctas;
                const unsigned g = ((unsigned)r % S) * ((unsigned)nseg_max % S) % S;
                k0 = (int)(((unsigned)cta + S - g) % S);
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

#ifdef MQA_DEBUG
// ---------------------------------------------------------------- debug builds
// Compiled only with -DMQA_DEBUG. A consumer checks every work-table entry as
// it walks the table (debug_check_unit); once every role is done the kernel
// checks that the roles walked the same units and tiles and that each
// pipeline barrier ended in the phase its use count predicts (debug_phases).
// A failure raises MQA_STATUS_DEBUG_INVARIANT; the work itself is unchanged.
// Nothing here runs after an abort, when the pipeline stopped part way.

// What one consumer has seen so far, and this CTA's schedule range.
struct DebugWalk {
    int units = 0, tiles = 0, rows = 0, last_b = -1, last_j = -1;
    int rs = 0, js = 0, re = 0, je = 0;
};

__device__ __forceinline__ void debug_walk_begin(const KernelArgs& a, int cta, DebugWalk& w) {
    w.rs = ptx::ld_cg(a.schedule + 2 * cta);
    w.js = ptx::ld_cg(a.schedule + 2 * cta + 1);
    w.re = ptx::ld_cg(a.schedule + 2 * cta + 2);
    w.je = ptx::ld_cg(a.schedule + 2 * cta + 3);
}

// Unit (row d.b, unit j = d.t0 / 256) must be the next unit of this CTA's
// range in row order: inside [entry cta, entry cta + 1), the row's effective
// context, its tiles numbered on from the previous unit's, and the row-start
// flag and row sequence number of `info` consistent with the rows seen.
__device__ __forceinline__ void debug_check_unit(const KernelArgs& a, const UnitDesc& d, int info,
                                                 DebugWalk& w) {
    const int j = d.t0 / kUnit;
    bool ok = d.b >= 0 && d.b < a.batch && d.t0 >= 0 && d.t0 % kUnit == 0 && d.t0 < d.ctx &&
              d.tile == w.tiles;
    if (ok) ok = d.ctx == min(max(ptx::ld_cg(a.context_lens + d.b), 0), a.ctx_cap);
    ok = ok && (d.b > w.rs || (d.b == w.rs && j >= w.js)) && (d.b < w.re || (d.b == w.re && j < w.je));
    if (info & 1) {
        ok = ok && d.b > w.last_b && (info >> 1) == w.rows && j == (d.b == w.rs ? w.js : 0);
        ++w.rows;
    } else {
        ok = ok && d.b == w.last_b && (info >> 1) == w.rows - 1 && j == w.last_j + 1;
    }
    if (!ok) raise_status(a, MQA_STATUS_DEBUG_INVARIANT);
    w.last_b = d.b;
    w.last_j = j;
    ++w.units;
    w.tiles += unit_tiles(d);
}

// Of `total` uses dealt round robin over m places, how many place i gets.
__device__ __forceinline__ int debug_share(int total, int i, int m) {
    return total / m + (i < total % m ? 1 : 0);
}

// After every role is done: `bar` has completed exactly n phases (modulo 2,
// which is what its parity shows): phase n - 1 is complete (waited for up to
// 1 ms, for tensor-core commits still on their way) and phase n is not.
__device__ __forceinline__ bool debug_phases(uint64_t* bar, int n) {
    if (n > 0) {
        const uint64_t t0 = ptx::globaltimer();
        while (!ptx::mbar_test_wait(bar, (uint32_t)(n - 1) & 1))
            if (ptx::globaltimer() - t0 > 1000000) return false;
    }
    return !ptx::mbar_test_wait(bar, (uint32_t)n & 1);
}

#endif
// Validate mode: does the schedule entry pair of `cta` match the current
// context_lens? (the reuse rule: a schedule stays valid only while every
// ceil(ctx_b / 256) is unchanged). One warp recomputes the unit prefix sums at
// this CTA's two entries and the total; a mismatch raises
// MQA_STATUS_STALE_SCHEDULE. The work itself is not changed.
__device__ __forceinline__ void check_schedule(const KernelArgs& a, int cta, int lane) {
    const int rs = ptx::ld_cg(a.schedule + 2 * cta), js = ptx::ld_cg(a.schedule + 2 * cta + 1);
    const int re = ptx::ld_cg(a.schedule + 2 * cta + 2), je = ptx::ld_cg(a.schedule + 2 * cta + 3);
    long long total = 0, before_s = 0, before_e = 0;
    int us = 0, ue = 0;
    for (int b = lane; b < a.batch; b += 32) {
        const int u = units_of(max(ptx::ld_cg(a.context_lens + b), 0));
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
