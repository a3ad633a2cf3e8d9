// Top-k selection over the logits: the indexer's use of them (the page
// "[flashinfer] Blackwell 아키텍처를 위한 고성능 Paged MQA Logits 커널 도입",
// introduction: the DeepSeek sparse-attention indexer scores every cached
// token and sparse attention then reads the best-scoring ones).
//
// For every row (b, n): the k tokens t < ctx_{b,n} of largest logit (for equal
// logits the lower tokens; -0.0 and +0.0 are equal), listed by logit
// descending then token ascending, or (MQA_TOPK_BY_TOKEN) by token ascending;
// rows with fewer than k valid tokens are padded with -1.
//
// One CTA per row. Logits map to order-preserving 32-bit keys. The first read
// of a row finds its key range [kmin, kmax]; all keys share the bits above the
// highest bit where kmin and kmax differ, so the radix select (histograms in
// shared memory, a block suffix scan to pick the digit) starts there and takes
// 11 bits a level until it has the k-th largest key T and how many keys equal
// to T to take. Starting at the range rather than at bit 31 matters for real
// logits: sums of ReLU terms sit in a narrow positive range, where the top 11
// bits are nearly constant and would pile every key onto a few bins. Rows are
// read from global memory with 16-byte loads, eight per thread in flight for
// rows longer than 16384 (four, and two CTAs per SM, otherwise):
//   cached     rows of up to 16384 valid tokens: the first read keeps every
//              key in shared memory and the levels read them there;
//   candidates longer rows: once the keys on T's prefix fit in shared memory
//              (8192), one more read splits the row, in token order, into the
//              keys above the prefix (all taken, written to the result) and a
//              candidate list that the remaining levels read;
//   global     otherwise every level re-reads the row.
// The take runs in token order (block prefix sums), so by-token results need
// no sort; by-value results get a bitonic sort of (key, ~token) pairs.
#include <cuda_runtime.h>

#include <cstdint>

#include "mqa_logits.h"
#include "ptx.cuh"

namespace mqa {

constexpr int kTopkThreads = 512;
constexpr int kTopkBins = 2048;        // widest radix digit: 11 bits
static_assert(kTopkBins % kTopkThreads == 0, "threads own whole digits of a histogram");
constexpr int kTopkCacheKeys = 16384;  // 64 KB of keys (or 8192 candidates)
constexpr int kTopkMinSort = 64;       // one warp's segment: 2 elements a lane
constexpr int kTopkLongRow = 16384;    // rows longer than this read with kTopkUnrollLong
constexpr int kTopkUnrollLong = 8;     // 16-byte loads in flight a thread: one CTA per SM
constexpr int kTopkUnrollShort = 4;    // ... for shorter rows: two CTAs per SM
constexpr int kTopkMaxShards = MQA_TOPK_MERGE_MAX_SHARDS;
constexpr int kTopkClusterMinRow = 32768;  // rows of at least this many logits may be split
constexpr int kTopkMaxCluster = 4;
constexpr int kTopkSms = 148;             // B200

// Order-preserving map of fp32 to uint32 (larger value, larger key); -0.0
// maps like +0.0.
__device__ __forceinline__ uint32_t topk_key(float v) {
    uint32_t u = __float_as_uint(v);
    if (u == 0x80000000u) u = 0u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// (key, token) packed so that a larger value means earlier in value order.
__device__ __forceinline__ uint64_t topk_pack(uint32_t key, int t) {
    return ((uint64_t)key << 32) | (uint32_t)(~(uint32_t)t);
}
__device__ __forceinline__ int topk_token(uint64_t p) { return (int)(~(uint32_t)p); }

// Block-wide exclusive prefix sum of v over the CTA's threads (in thread
// order); `total` gets the sum. Uses ws[0..32] of shared memory.
__device__ __forceinline__ int block_exscan(int v, int* ws, int& total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int x = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += x;
    }
    if (lane == 31) ws[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int w = lane < nw ? ws[lane] : 0;
        int wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int x = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o) wi += x;
        }
        if (lane < nw) ws[lane] = wi - w;
        if (lane == 31) ws[32] = wi;
    }
    __syncthreads();
    const int ex = ws[warp] + incl - v;
    total = ws[32];
    __syncthreads();  // ws is reused by the next call
    return ex;
}

// The digit d of histogram hist[0, nb) with (count of digits > d) < remaining
// <= (count of digits >= d); returns d, sets remaining to how many of the
// keys with digit d are still to take and n_match to how many keys have digit
// d. No thread reads hist after the call returns. With per = max(nb / blockDim.x, 1),
// thread i owns the per digits from nb - 1 - i * per down (none once that is
// negative), so a prefix sum over threads is a suffix sum over digits. nb is
// a power of two, at most kTopkBins. Uniform over the CTA.
__device__ __forceinline__ int select_digit(const int* hist, int nb, int& remaining,
                                            int& n_match, int* ws, int* bcast) {
    constexpr int kMaxPer = kTopkBins / kTopkThreads;
    const int per = nb > (int)blockDim.x ? nb / (int)blockDim.x : 1;
    const int top = nb - 1 - (int)threadIdx.x * per;  // highest digit owned (< 0: none)
    int h[kMaxPer];
    int sum = 0;
#pragma unroll
    for (int j = 0; j < kMaxPer; ++j) {
        h[j] = (j < per && top - j >= 0) ? hist[top - j] : 0;
        sum += h[j];
    }
    int total;
    int above = block_exscan(sum, ws, total);  // count of digits > top
#pragma unroll
    for (int j = 0; j < kMaxPer; ++j) {
        if (j < per && top - j >= 0 && above < remaining && remaining <= above + h[j]) {
            bcast[0] = top - j;
            bcast[1] = remaining - above;
        }
        above += h[j];
    }
    __syncthreads();
    const int d = bcast[0];
    remaining = bcast[1];
    n_match = hist[d];
    __syncthreads();
    return d;
}

// Four consecutive tokens i..i+3 of a row (i a multiple of 4): keys and
// tokens, token -1 past the row's n valid ones.
struct Quad {
    uint32_t key[4];
    int tok[4];
};

__device__ __forceinline__ Quad load_cached(const uint32_t* keys, int i, int n) {
    Quad q;
    const uint4 k4 = i < n ? *reinterpret_cast<const uint4*>(keys + i) : make_uint4(0, 0, 0, 0);
    q.key[0] = k4.x, q.key[1] = k4.y, q.key[2] = k4.z, q.key[3] = k4.w;
#pragma unroll
    for (int e = 0; e < 4; ++e) q.tok[e] = i + e < n ? i + e : -1;
    return q;
}

__device__ __forceinline__ Quad load_cand(const uint64_t* cand, int i, int n) {
    Quad q;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const uint64_t p = i + e < n ? cand[i + e] : 0ull;
        q.key[e] = (uint32_t)(p >> 32);
        q.tok[e] = i + e < n ? topk_token(p) : -1;
    }
    return q;
}

// Visits entries [0, n) in chunks of 4 * blockDim.x, U chunks loaded before
// any is processed; thread j gets entries 4j..4j+3 of each chunk, so thread
// order within a chunk is entry order. `body(quad, i)` is called by every
// thread for every chunk (uniformly: it may hold block barriers).
template <int U, class Load, class Body>
__device__ __forceinline__ void for_quads(int n, Load load, Body body) {
    const int per = 4 * (int)blockDim.x;
    for (int base = 0; base < n; base += U * per) {
        Quad q[U];
#pragma unroll
        for (int u = 0; u < U; ++u) q[u] = load(base + u * per + 4 * (int)threadIdx.x);
#pragma unroll
        for (int u = 0; u < U; ++u)
            if (base + u * per < n) body(q[u], base + u * per + 4 * (int)threadIdx.x);
    }
}

// for_quads over a row of n fp32 logits in global memory: all U loads of a
// thread (16 bytes each when the row is 16-byte aligned, else four scalar
// loads) are issued before any is converted to keys, so U loads are in
// flight per thread.
template <int U, class Body>
__device__ __forceinline__ void for_quads_global(const float* __restrict__ x, bool vec, int n,
                                                 Body body) {
    const int per = 4 * (int)blockDim.x;
    for (int base = 0; base < n; base += U * per) {
        float4 raw[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int i = base + u * per + 4 * (int)threadIdx.x;
            raw[u] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (vec && i + 3 < n) raw[u] = __ldg(reinterpret_cast<const float4*>(x + i));
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int i = base + u * per + 4 * (int)threadIdx.x;
            if (!(vec && i + 3 < n) && i < n) {  // unaligned row or its last quad
                raw[u].x = __ldg(x + i);
                if (i + 1 < n) raw[u].y = __ldg(x + i + 1);
                if (i + 2 < n) raw[u].z = __ldg(x + i + 2);
                if (i + 3 < n) raw[u].w = __ldg(x + i + 3);
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int i = base + u * per + 4 * (int)threadIdx.x;
            if (base + u * per < n) {
                Quad q;
                q.key[0] = topk_key(raw[u].x);
                q.key[1] = topk_key(raw[u].y);
                q.key[2] = topk_key(raw[u].z);
                q.key[3] = topk_key(raw[u].w);
#pragma unroll
                for (int e = 0; e < 4; ++e) q.tok[e] = i + e < n ? i + e : -1;
                body(q, i);
            }
        }
    }
}

// Bitonic compare-exchange of this lane's element (global index i, value v)
// with the element i ^ stride held by lane ^ stride (stride < 32). The pair
// sorts descending when its lower index has bit `size` clear.
__device__ __forceinline__ uint64_t bitonic_lane_step(uint64_t v, int i, int stride, int size) {
    const uint64_t p = __shfl_xor_sync(0xffffffffu, v, stride);
    const bool lower = (i & stride) == 0;
    const bool desc = ((i & ~stride) & size) == 0;
    const uint64_t hi = v > p ? v : p, lo = v > p ? p : v;
    return (lower == desc) ? hi : lo;
}

// Strides 32, 16, ..., 1 of bitonic merge step `size` on one 64-element
// segment held as a (index base + lane) and b (base + 32 + lane).
__device__ __forceinline__ void bitonic_warp_merge(uint64_t& a, uint64_t& b, int base, int lane,
                                                   int size, int top_stride) {
    if (top_stride >= 32) {  // in-thread pair (base + lane, base + lane + 32)
        const bool desc = ((base + lane) & size) == 0;
        if (desc ? (a < b) : (a > b)) {
            const uint64_t t = a;
            a = b;
            b = t;
        }
    }
    for (int s = top_stride < 16 ? top_stride : 16; s > 0; s >>= 1) {
        a = bitonic_lane_step(a, base + lane, s, size);
        b = bitonic_lane_step(b, base + 32 + lane, s, size);
    }
}

// Descending bitonic sort of sel[0, len), len a power of two >= 64. Warp w
// owns 64-element segments w, w + nwarps, ...: lane l holds elements l and
// l + 32 of a segment for the strides below 64.
__device__ void bitonic_sort_desc(uint64_t* sel, int len) {
    const int tid = threadIdx.x, nthr = blockDim.x, lane = tid & 31, warp = tid >> 5;
    const int nseg = len >> 6, nwarps = nthr >> 5;
    for (int seg = warp; seg < nseg; seg += nwarps) {
        const int base = seg << 6;
        uint64_t a = sel[base + lane], bv = sel[base + 32 + lane];
        for (int size = 2; size <= 64; size <<= 1) bitonic_warp_merge(a, bv, base, lane, size, size >> 1);
        sel[base + lane] = a;
        sel[base + 32 + lane] = bv;
    }
    __syncthreads();
    for (int size = 128; size <= len; size <<= 1) {
        for (int stride = size >> 1; stride >= 64; stride >>= 1) {
            for (int i = tid; i < (len >> 1); i += nthr) {
                const int lo = 2 * i - (i & (stride - 1));
                const int hi = lo + stride;
                const uint64_t a = sel[lo], bb = sel[hi];
                const bool desc = (lo & size) == 0;
                if (desc ? (a < bb) : (a > bb)) {
                    sel[lo] = bb;
                    sel[hi] = a;
                }
            }
            __syncthreads();
        }
        for (int seg = warp; seg < nseg; seg += nwarps) {
            const int base = seg << 6;
            uint64_t a = sel[base + lane], bv = sel[base + 32 + lane];
            bitonic_warp_merge(a, bv, base, lane, size, 32);
            sel[base + lane] = a;
            sel[base + 32 + lane] = bv;
        }
        __syncthreads();
    }
}

// Number of entries of sel[0, n) (ascending by token) with token < t.
__device__ __forceinline__ int count_tokens_below(const uint64_t* sel, int n, int t) {
    int lo = 0, hi = n;
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (topk_token(sel[mid]) < t) lo = mid + 1;
        else hi = mid;
    }
    return lo;
}

// Value of a key (the inverse of topk_key; -0.0 comes back as +0.0).
__device__ __forceinline__ float key_value(uint32_t key) {
    return __uint_as_float((key & 0x80000000u) ? (key ^ 0x80000000u) : ~key);
}

// Arguments of one launch. Row mode: rows of logits [rows][L] with the valid
// prefix of each given by context_lens and next_n. Merge mode (shards > 0):
// row r's entries are the shards' lists [shards][rows][k_in] of (value,
// local token) pairs, token -1 for an empty slot; a shard's tokens are
// ascending and shard s's global tokens are local + offsets[s], increasing
// with s, so the concatenation in shard order is in global token order.
struct TopkParams {
    const float* logits;
    const int32_t* context_lens;
    const int32_t* cand_tokens;
    int32_t* out;    // [rows][k]
    float* values;   // [rows][k] or null
    int next_n, L, k, region_words, by_token;
    int rows, shards, k_in;
    int offsets[kTopkMaxShards];
};

// U: 16-byte global loads in flight per thread; the short-row instance is
// held to 64 registers so that two CTAs share an SM.
template <int U>
__global__ void __launch_bounds__(kTopkThreads, U == kTopkUnrollShort ? 2 : 1)
    topk_kernel(const __grid_constant__ TopkParams p) {
    extern __shared__ uint64_t sel[];  // [sort_n] packed (key, token), then the region
    __shared__ int hist[2][kTopkBins];  // one level's histogram, the next one's zeroed
    __shared__ int ws[33];
    __shared__ int bcast[2];
    __shared__ uint32_t ubc[2];  // row key range

    ptx::griddep_launch_dependents();
    ptx::griddep_wait();  // the logits may come from the previous kernel

    const int k = p.k, tid = threadIdx.x, nthr = blockDim.x, row = blockIdx.x;
    int sort_n = kTopkMinSort;
    while (sort_n < k) sort_n <<= 1;
    uint32_t* keys = reinterpret_cast<uint32_t*>(sel + sort_n);  // cached keys [region_words]
    uint64_t* cand = sel + sort_n;                                // or candidates [region_words / 2]
    int32_t* o = p.out + (int64_t)row * k;
    float* vo = p.values ? p.values + (int64_t)row * k : nullptr;
    auto emit = [&](int pos, uint32_t key, int t) {
        o[pos] = t;
        if (vo) vo[pos] = key_value(key);
    };
    auto pad = [&](int pos) {
        o[pos] = -1;
        if (vo) vo[pos] = __uint_as_float(0xff800000u);  // -inf
    };

    const float* x = nullptr;
    bool vec = false;
    int cbn;       // entries of the row
    int src;       // 0 global row, 1 cached keys, 2 candidate list
    if (p.shards > 0) {
        // merge mode: compact the valid entries, in shard order, into cand[]
        const int E = p.shards * p.k_in;
        auto mload = [&](int i) {
            Quad q;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                q.key[e] = 0u;
                q.tok[e] = -1;
                if (i + e < E) {
                    const int sh = (i + e) / p.k_in, j = i + e - sh * p.k_in;
                    const int64_t at = ((int64_t)sh * p.rows + row) * p.k_in + j;
                    const int t = __ldg(p.cand_tokens + at);
                    if (t >= 0) {
                        q.key[e] = topk_key(__ldg(p.logits + at));
                        q.tok[e] = t + p.offsets[sh];
                    }
                }
            }
            return q;
        };
        int base = 0;
        for_quads<1>(E, mload, [&](const Quad& q, int) {
            int nv = 0;
#pragma unroll
            for (int e = 0; e < 4; ++e) nv += q.tok[e] >= 0;
            int tot;
            int pos = base + block_exscan(nv, ws, tot);
#pragma unroll
            for (int e = 0; e < 4; ++e)
                if (q.tok[e] >= 0) cand[pos++] = topk_pack(q.key[e], q.tok[e]);
            base += tot;
        });
        __syncthreads();
        cbn = base;
        src = 2;
    } else {
        const int next_n = p.next_n, L = p.L;
        const int b = row / next_n, n = row - b * next_n;
        int c = __ldg(p.context_lens + b);
        c = c < 0 ? 0 : (c > L ? L : c);
        cbn = c - next_n + 1 + n;
        cbn = cbn < 0 ? 0 : (cbn > c ? c : cbn);
        x = p.logits + (int64_t)row * L;
        vec = (reinterpret_cast<uintptr_t>(x) & 15) == 0;
        src = cbn <= p.region_words ? 1 : 0;
    }
    const int m = cbn < k ? cbn : k;  // entries taken

    if (cbn <= k) {  // every valid entry is taken
        if (p.by_token) {
            for (int i = tid; i < k; i += nthr) {
                if (i >= cbn) pad(i);
                else if (src == 2) emit(i, (uint32_t)(cand[i] >> 32), topk_token(cand[i]));
                else emit(i, vo ? topk_key(__ldg(x + i)) : 0u, i);
            }
            return;
        }
        if (src == 2) {
            for (int i = tid; i < cbn; i += nthr) sel[i] = cand[i];
        } else {
            for_quads_global<U>(x, vec, cbn, [&](const Quad& q, int) {
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    if (q.tok[e] >= 0) sel[q.tok[e]] = topk_pack(q.key[e], q.tok[e]);
            });
        }
    } else {
        const int cand_cap = p.region_words / 2;
        auto cload = [&](int i) { return load_cand(cand, i, cbn); };
        // the range [kmin, kmax] of the row's keys (for a row in global
        // memory this is its first read, which also fills the key cache)
        if (tid == 0) {
            ubc[0] = 0xffffffffu;
            ubc[1] = 0u;
        }
        for (int i = tid; i < kTopkBins; i += nthr) hist[0][i] = 0;  // the first level's
        __syncthreads();
        uint32_t lmin = 0xffffffffu, lmax = 0u;
        auto range = [&](const Quad& q, int i) {
            if (src == 1 && i < cbn)  // i + 3 < cbn rounded up to 4 <= region_words
                *reinterpret_cast<uint4*>(keys + i) = make_uint4(q.key[0], q.key[1], q.key[2], q.key[3]);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                if (q.tok[e] < 0) continue;
                lmin = q.key[e] < lmin ? q.key[e] : lmin;
                lmax = q.key[e] > lmax ? q.key[e] : lmax;
            }
        };
        if (src == 2) for_quads<1>(cbn, cload, range);
        else for_quads_global<U>(x, vec, cbn, range);
        lmin = __reduce_min_sync(0xffffffffu, lmin);
        lmax = __reduce_max_sync(0xffffffffu, lmax);
        if ((tid & 31) == 0) {
            atomicMin(&ubc[0], lmin);
            atomicMax(&ubc[1], lmax);
        }
        __syncthreads();
        const uint32_t kmin = ubc[0], kmax = ubc[1];
        if (kmin == kmax) {
            // all keys equal: the first k entries, in either order
            for (int i = tid; i < k; i += nthr) emit(i, kmin, src == 2 ? topk_token(cand[i]) : i);
            return;
        }
        // Digits start at the highest bit where keys differ (all keys share
        // the bits above it), 11 bits a level: level j covers bits
        // [s_lo, s) and narrows (prefix, mask) to T's bits >= s_lo.
        const int hb = 31 - __clz(kmin ^ kmax);
        uint32_t mask = hb == 31 ? 0u : (0xffffffffu << (hb + 1));
        uint32_t prefix = kmin & mask;
        int remaining = k;
        int n_src = cbn;    // entries of the current source
        int n_above = 0;    // after a split: entries taken before the list
        auto lload = [&](int i) { return load_cand(cand, i, n_src); };
        auto kload = [&](int i) { return load_cached(keys, i, cbn); };
        bool exact = true;  // false: every key of T's last bin is taken (see below)
        for (int s = hb + 1, lv = 0; s > 0; ++lv) {
            const int s_lo = s > 11 ? s - 11 : 0;
            const int nb = 1 << (s - s_lo);
            int* h = hist[lv & 1];
            int* h_next = hist[(lv + 1) & 1];  // last read inside the previous level's select
            auto hist_body = [&](const Quad& q, int) {
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    if (q.tok[e] >= 0 && (q.key[e] & mask) == prefix)
                        atomicAdd(&h[(q.key[e] >> s_lo) & (nb - 1)], 1);
            };
            if (src == 0) for_quads_global<U>(x, vec, cbn, hist_body);
            else if (src == 1) for_quads<1>(cbn, kload, hist_body);
            else for_quads<1>(n_src, lload, hist_body);
            for (int i = tid; i < kTopkBins; i += nthr) h_next[i] = 0;
            __syncthreads();
            int n_match;
            const int d = select_digit(h, nb, remaining, n_match, ws, bcast);
            prefix |= (uint32_t)d << s_lo;
            mask = 0xffffffffu << s_lo;
            s = s_lo;
            if (s > 0 && remaining == n_match) {
                // every key on the prefix is taken: the threshold is the
                // prefix itself, the lower bits need no more levels
                exact = false;
                break;
            }
            if (src == 0 && s > 0 && n_match <= cand_cap) {
                // split the row, in token order: keys above the prefix ->
                // sel[0, n_above) (all taken); keys on it -> cand[0, n_match)
                n_above = k - remaining;
                int base_a = 0, base_c = 0;
                for_quads_global<U>(x, vec, cbn, [&](const Quad& q, int) {
                    int na = 0, nc = 0;
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        if (q.tok[e] < 0) continue;
                        const uint32_t km = q.key[e] & mask;
                        na += km > prefix;
                        nc += km == prefix;
                    }
                    int tot;
                    const int ex = block_exscan(na | (nc << 16), ws, tot);
                    int pa = base_a + (ex & 0xffff), pc = base_c + (ex >> 16);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        if (q.tok[e] < 0) continue;
                        const uint32_t km = q.key[e] & mask;
                        if (km > prefix) sel[pa++] = topk_pack(q.key[e], q.tok[e]);
                        else if (km == prefix) cand[pc++] = topk_pack(q.key[e], q.tok[e]);
                    }
                    base_a += tot & 0xffff;
                    base_c += tot >> 16;
                });
                __syncthreads();
                src = 2;
                n_src = n_match;
            }
        }
        // keys > T are all taken, and the first take_eq keys == T. When the
        // loop stopped early, the taken keys are exactly those >= prefix (its
        // low bits are zero); prefix > 0 there, since otherwise all cbn > k
        // keys would be taken.
        const uint32_t T = exact ? prefix : prefix - 1u;
        const int take_eq = exact ? remaining : 0;
        const bool to_sel = src == 2 || !p.by_token;

        // take, in token order: a key is taken if > T, or == T among the first
        // take_eq of those; its place among the taken ones is the count of
        // earlier keys > T plus min(earlier keys == T, take_eq).
        int base_gt = 0, base_eq = 0;
        auto take = [&](const Quad& q, int) {
            int ng = 0, ne = 0;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                if (q.tok[e] < 0) continue;
                ng += q.key[e] > T;
                ne += q.key[e] == T;
            }
            int tot;
            const int ex = block_exscan(ng | (ne << 16), ws, tot);
            int g = base_gt + (ex & 0xffff), eq = base_eq + (ex >> 16);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                if (q.tok[e] < 0) continue;
                const bool is_gt = q.key[e] > T, is_eq = q.key[e] == T;
                if (is_gt || (is_eq && eq < take_eq)) {
                    const int pos = n_above + g + (eq < take_eq ? eq : take_eq);
                    if (to_sel) sel[pos] = topk_pack(q.key[e], q.tok[e]);
                    else emit(pos, q.key[e], q.tok[e]);
                }
                g += is_gt;
                eq += is_eq;
            }
            base_gt += tot & 0xffff;
            base_eq += tot >> 16;
        };
        if (src == 0) for_quads_global<U>(x, vec, cbn, take);
        else if (src == 1) for_quads<1>(cbn, kload, take);
        else for_quads<1>(n_src, lload, take);
        __syncthreads();

        if (p.by_token) {
            if (to_sel) {
                // merge sel[0, n_above) and sel[n_above, k), both by token
                for (int i = tid; i < k; i += nthr) {
                    const uint64_t e = sel[i];
                    const int t = topk_token(e);
                    const int pos = i < n_above
                                        ? i + count_tokens_below(sel + n_above, k - n_above, t)
                                        : (i - n_above) + count_tokens_below(sel, n_above, t);
                    emit(pos, (uint32_t)(e >> 32), t);
                }
            }
            return;  // k taken, none padded
        }
    }

    // by value: sort the m taken entries (padding sorts last), then write
    int len = kTopkMinSort;
    while (len < m) len <<= 1;
    for (int i = m + tid; i < len; i += nthr) sel[i] = 0ull;
    __syncthreads();
    bitonic_sort_desc(sel, len);
    for (int i = tid; i < k; i += nthr) {
        if (i < m) emit(i, (uint32_t)(sel[i] >> 32), topk_token(sel[i]));
        else pad(i);
    }
}

// ---------------------------------------------------------------- cluster split
// A row that one CTA would take alone while SMs sit idle (few, long rows) is
// split over a cluster of C CTAs: rank r reads the row's tokens
// [r * per, (r + 1) * per). Every cluster-wide quantity (the key range, each
// level's histogram, the counts before the take, the by-value gather) goes
// through distributed shared memory behind cluster barriers. Every rank
// derives its control flow from those cluster-wide values only, so all ranks
// pass the same barriers in the same order; a rank with no tokens takes part
// with zero counts. Each rank keeps the single-CTA machinery for its own
// range (cached keys, or global re-reads with a local split into candidates).

__device__ __forceinline__ uint32_t cl_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t cl_size() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
    return r;
}
// All threads of all CTAs of the cluster; orders shared-memory writes before
// the barrier with reads after it, cluster-wide.
__device__ __forceinline__ void cl_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;"
                 ::: "memory");
}
// Address of this CTA's shared variable `p` in the shared memory of `rank`.
__device__ __forceinline__ uint32_t cl_map(const void* p, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(ptx::smem_u32(p)), "r"(rank));
    return r;
}
__device__ __forceinline__ int cl_ld(uint32_t a) {
    int v;
    asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(a) : "memory");
    return v;
}
__device__ __forceinline__ void cl_st64(uint32_t a, uint64_t v) {
    asm volatile("st.shared::cluster.u64 [%0], %1;" ::"r"(a), "l"(v) : "memory");
}

// select_digit over the sum of the C ranks' histograms `hist` (the same
// shared variable in every rank). Also returns this rank's own count of keys
// with digits above d (above_loc) and with digit d (match_loc).
__device__ __forceinline__ int select_digit_cluster(const int* hist, int nb, int C, int& remaining,
                                                    int& n_match, int& above_loc, int& match_loc,
                                                    int* ws, int* bcast, int* red) {
    constexpr int kMaxPer = kTopkBins / kTopkThreads;
    const int per = nb > (int)blockDim.x ? nb / (int)blockDim.x : 1;
    const int top = nb - 1 - (int)threadIdx.x * per;
    int h[kMaxPer], hl[kMaxPer];
    int v[kMaxPer][kTopkMaxCluster];
    // every remote read issued before any is used, so they are in flight together
#pragma unroll
    for (int j = 0; j < kMaxPer; ++j) {
        const bool own = j < per && top - j >= 0;
        hl[j] = own ? hist[top - j] : 0;
#pragma unroll
        for (int r = 0; r < kTopkMaxCluster; ++r)
            v[j][r] = (own && r < C) ? cl_ld(cl_map(hist + (top - j), (uint32_t)r)) : 0;
    }
    int sum = 0;
#pragma unroll
    for (int j = 0; j < kMaxPer; ++j) {
        h[j] = 0;
#pragma unroll
        for (int r = 0; r < kTopkMaxCluster; ++r) h[j] += v[j][r];
        sum += h[j];
    }
    int total;
    int above = block_exscan(sum, ws, total);
#pragma unroll
    for (int j = 0; j < kMaxPer; ++j) {
        if (j < per && top - j >= 0 && above < remaining && remaining <= above + h[j]) {
            bcast[0] = top - j;
            bcast[1] = remaining - above;
            bcast[2] = h[j];
        }
        above += h[j];
    }
    if (threadIdx.x == 0) {
        red[0] = 0;
        red[1] = 0;
    }
    __syncthreads();
    const int d = bcast[0];
    int a_loc = 0, m_loc = 0;
#pragma unroll
    for (int j = 0; j < kMaxPer; ++j) {
        if (j < per && top - j >= 0) {
            if (top - j > d) a_loc += hl[j];
            if (top - j == d) m_loc += hl[j];
        }
    }
    a_loc = __reduce_add_sync(0xffffffffu, a_loc);
    m_loc = __reduce_add_sync(0xffffffffu, m_loc);
    if ((threadIdx.x & 31) == 0) {
        atomicAdd(&red[0], a_loc);
        atomicAdd(&red[1], m_loc);
    }
    __syncthreads();
    remaining = bcast[1];
    n_match = bcast[2];
    above_loc = red[0];
    match_loc = red[1];
    __syncthreads();  // bcast and red are reused by the next call
    return d;
}

template <int U>
__global__ void __launch_bounds__(kTopkThreads, 2)
    topk_cluster_kernel(const __grid_constant__ TopkParams p) {
    extern __shared__ uint64_t sel[];  // [sort_n] packed (key, token), then the region
    __shared__ int hist[2][kTopkBins];
    __shared__ int ws[33];
    __shared__ int bcast[3];
    __shared__ int red[2];
    __shared__ uint32_t ubc[2];  // this rank's key range
    __shared__ int cnt[2];       // this rank's keys > T and == T
    __shared__ int place[2];     // this rank's first output slot and its share of keys == T

    ptx::griddep_launch_dependents();
    ptx::griddep_wait();  // the logits may come from the previous kernel

    const int C = (int)cl_size(), rank = (int)cl_rank();
    const int k = p.k, tid = threadIdx.x, nthr = blockDim.x, row = blockIdx.x / C;
    int sort_n = kTopkMinSort;
    while (sort_n < k) sort_n <<= 1;
    uint32_t* keys = reinterpret_cast<uint32_t*>(sel + sort_n);
    uint64_t* cand = sel + sort_n;
    int32_t* o = p.out + (int64_t)row * k;
    float* vo = p.values ? p.values + (int64_t)row * k : nullptr;
    auto emit = [&](int pos, uint32_t key, int t) {
        o[pos] = t;
        if (vo) vo[pos] = key_value(key);
    };
    auto pad = [&](int pos) {
        o[pos] = -1;
        if (vo) vo[pos] = __uint_as_float(0xff800000u);  // -inf
    };

    const int next_n = p.next_n, L = p.L;
    const int b = row / next_n, n = row - b * next_n;
    int c = __ldg(p.context_lens + b);
    c = c < 0 ? 0 : (c > L ? L : c);
    int cbn = c - next_n + 1 + n;
    cbn = cbn < 0 ? 0 : (cbn > c ? c : cbn);
    const float* xrow = p.logits + (int64_t)row * L;
    const bool vec = (reinterpret_cast<uintptr_t>(xrow) & 15) == 0;
    // this rank's tokens [lo, hi): whole quads, so its loads stay 16-byte aligned
    const int per = ((cbn + C - 1) / C + 3) & ~3;
    const int lo = min(rank * per, cbn), hi = min(lo + per, cbn), nl = hi - lo;
    const float* x = xrow + lo;
    int src = nl <= p.region_words ? 1 : 0;  // 0 global, 1 cached keys, 2 candidates

    if (cbn <= k) {
        // every valid entry is taken
        if (p.by_token) {
            for (int i = lo + tid; i < hi; i += nthr) emit(i, vo ? topk_key(__ldg(xrow + i)) : 0u, i);
            if (rank == 0)
                for (int i = cbn + tid; i < k; i += nthr) pad(i);
        } else {
            // gather into rank 0, which sorts
            for (int i = lo + tid; i < hi; i += nthr)
                cl_st64(cl_map(sel + i, 0), topk_pack(topk_key(__ldg(xrow + i)), i));
            cl_sync();
            if (rank == 0) {
                int len = kTopkMinSort;
                while (len < cbn) len <<= 1;
                for (int i = cbn + tid; i < len; i += nthr) sel[i] = 0ull;
                __syncthreads();
                bitonic_sort_desc(sel, len);
                for (int i = tid; i < k; i += nthr) {
                    if (i < cbn) emit(i, (uint32_t)(sel[i] >> 32), topk_token(sel[i]));
                    else pad(i);
                }
            }
        }
        cl_sync();  // no rank leaves while another may still touch its shared memory
        return;
    }

    // the key range: each rank's, then the cluster's
    if (tid == 0) {
        ubc[0] = 0xffffffffu;
        ubc[1] = 0u;
    }
    for (int i = tid; i < kTopkBins; i += nthr) hist[0][i] = 0;
    __syncthreads();
    uint32_t lmin = 0xffffffffu, lmax = 0u;
    auto range = [&](const Quad& q, int i) {
        if (src == 1 && i < nl)
            *reinterpret_cast<uint4*>(keys + i) = make_uint4(q.key[0], q.key[1], q.key[2], q.key[3]);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            if (q.tok[e] < 0) continue;
            lmin = q.key[e] < lmin ? q.key[e] : lmin;
            lmax = q.key[e] > lmax ? q.key[e] : lmax;
        }
    };
    for_quads_global<U>(x, vec, nl, range);
    lmin = __reduce_min_sync(0xffffffffu, lmin);
    lmax = __reduce_max_sync(0xffffffffu, lmax);
    if ((tid & 31) == 0) {
        atomicMin(&ubc[0], lmin);
        atomicMax(&ubc[1], lmax);
    }
    __syncthreads();
    cl_sync();
    uint32_t kmin = 0xffffffffu, kmax = 0u;
    for (int r = 0; r < C; ++r) {
        const uint32_t a = (uint32_t)cl_ld(cl_map(&ubc[0], (uint32_t)r));
        const uint32_t z = (uint32_t)cl_ld(cl_map(&ubc[1], (uint32_t)r));
        kmin = a < kmin ? a : kmin;
        kmax = z > kmax ? z : kmax;
    }
    if (kmin == kmax) {
        // all keys equal: the first k tokens, in either order
        for (int i = lo + tid; i < min(hi, k); i += nthr) emit(i, kmin, i);
        cl_sync();
        return;
    }

    const int cand_cap = p.region_words / 2;
    const int hb = 31 - __clz(kmin ^ kmax);
    uint32_t mask = hb == 31 ? 0u : (0xffffffffu << (hb + 1));
    uint32_t prefix = kmin & mask;
    int remaining = k;
    int n_src = nl;
    int n_above = 0;    // after a local split: this rank's keys taken before its list
    int above_acc = 0;  // this rank's keys above the chosen digits so far (all > T)
    int match_loc = 0;  // this rank's keys on the current prefix
    auto lload = [&](int i) { return load_cand(cand, i, n_src); };
    auto kload = [&](int i) { return load_cached(keys, i, nl); };
    bool exact = true;
    for (int s = hb + 1, lv = 0; s > 0; ++lv) {
        const int s_lo = s > 11 ? s - 11 : 0;
        const int nb = 1 << (s - s_lo);
        int* h = hist[lv & 1];
        int* h_next = hist[(lv + 1) & 1];
        auto hist_body = [&](const Quad& q, int) {
#pragma unroll
            for (int e = 0; e < 4; ++e)
                if (q.tok[e] >= 0 && (q.key[e] & mask) == prefix)
                    atomicAdd(&h[(q.key[e] >> s_lo) & (nb - 1)], 1);
        };
        if (src == 0) for_quads_global<U>(x, vec, nl, hist_body);
        else if (src == 1) for_quads<1>(nl, kload, hist_body);
        else for_quads<1>(n_src, lload, hist_body);
        __syncthreads();
        cl_sync();  // every rank's h is complete; nobody reads h_next any more
        for (int i = tid; i < kTopkBins; i += nthr) h_next[i] = 0;
        int n_match, a_loc;
        const int d = select_digit_cluster(h, nb, C, remaining, n_match, a_loc, match_loc, ws,
                                           bcast, red);
        above_acc += a_loc;
        prefix |= (uint32_t)d << s_lo;
        mask = 0xffffffffu << s_lo;
        s = s_lo;
        if (s > 0 && remaining == n_match) {
            exact = false;  // every key on the prefix is taken (cluster-wide)
            break;
        }
        if (src == 0 && s > 0 && match_loc <= cand_cap) {
            // local split, in token order: keys above the prefix -> sel (all
            // taken), keys on it -> cand
            n_above = above_acc;
            int base_a = 0, base_c = 0;
            for_quads_global<U>(x, vec, nl, [&](const Quad& q, int) {
                int na = 0, nc = 0;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    if (q.tok[e] < 0) continue;
                    const uint32_t km = q.key[e] & mask;
                    na += km > prefix;
                    nc += km == prefix;
                }
                int tot;
                const int ex = block_exscan(na | (nc << 16), ws, tot);
                int pa = base_a + (ex & 0xffff), pc = base_c + (ex >> 16);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    if (q.tok[e] < 0) continue;
                    const uint32_t km = q.key[e] & mask;
                    if (km > prefix) sel[pa++] = topk_pack(q.key[e], lo + q.tok[e]);
                    else if (km == prefix) cand[pc++] = topk_pack(q.key[e], lo + q.tok[e]);
                }
                base_a += tot & 0xffff;
                base_c += tot >> 16;
            });
            __syncthreads();
            src = 2;
            n_src = match_loc;
        }
    }
    const uint32_t T = exact ? prefix : prefix - 1u;
    const int take_eq = exact ? remaining : 0;

    // this rank's keys > T and == T, then its place in the cluster's output
    if (tid == 0) {
        cnt[0] = exact ? above_acc : above_acc + match_loc;
        cnt[1] = exact ? match_loc : 0;
    }
    __syncthreads();
    cl_sync();
    if (tid == 0) {
        int pos = 0, eq_before = 0, my_eq = 0;
        for (int r = 0; r < C; ++r) {
            const int gt = cl_ld(cl_map(&cnt[0], (uint32_t)r));
            const int ne = cl_ld(cl_map(&cnt[1], (uint32_t)r));
            const int te = max(0, min(ne, take_eq - eq_before));
            if (r == rank) {
                place[0] = pos;
                my_eq = te;
            }
            pos += gt + te;
            eq_before += ne;
        }
        place[1] = my_eq;
    }
    __syncthreads();
    const int P = place[0], take_eq_r = place[1];

    // take this rank's keys in token order; local slots n_above + g + min(eq, take_eq_r)
    int base_gt = 0, base_eq = 0;
    const bool to_sel = src == 2 || !p.by_token;
    auto take = [&](const Quad& q, int) {
        int ng = 0, ne = 0;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            if (q.tok[e] < 0) continue;
            ng += q.key[e] > T;
            ne += q.key[e] == T;
        }
        int tot;
        const int ex = block_exscan(ng | (ne << 16), ws, tot);
        int g = base_gt + (ex & 0xffff), eq = base_eq + (ex >> 16);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            if (q.tok[e] < 0) continue;
            const bool is_gt = q.key[e] > T, is_eq = q.key[e] == T;
            if (is_gt || (is_eq && eq < take_eq_r)) {
                const int pos = n_above + g + (eq < take_eq_r ? eq : take_eq_r);
                const int t = src == 2 ? q.tok[e] : lo + q.tok[e];
                if (to_sel) sel[pos] = topk_pack(q.key[e], t);
                else emit(P + pos, q.key[e], t);
            }
            g += is_gt;
            eq += is_eq;
        }
        base_gt += tot & 0xffff;
        base_eq += tot >> 16;
    };
    if (src == 0) for_quads_global<U>(x, vec, nl, take);
    else if (src == 1) for_quads<1>(nl, kload, take);
    else for_quads<1>(n_src, lload, take);
    __syncthreads();
    const int mine = cnt[0] + take_eq_r;  // entries this rank takes

    if (p.by_token) {
        if (to_sel) {
            // merge sel[0, n_above) and sel[n_above, mine), both by token
            for (int i = tid; i < mine; i += nthr) {
                const uint64_t e = sel[i];
                const int t = topk_token(e);
                const int pos = i < n_above
                                    ? i + count_tokens_below(sel + n_above, mine - n_above, t)
                                    : (i - n_above) + count_tokens_below(sel, n_above, t);
                emit(P + pos, (uint32_t)(e >> 32), t);
            }
        }
    } else {
        // gather every rank's entries into rank 0's sort buffer, which sorts
        __syncthreads();
        if (rank != 0)
            for (int i = tid; i < mine; i += nthr) cl_st64(cl_map(sel + P + i, 0), sel[i]);
        cl_sync();
        if (rank == 0) {
            int len = kTopkMinSort;
            while (len < k) len <<= 1;
            for (int i = k + tid; i < len; i += nthr) sel[i] = 0ull;
            __syncthreads();
            bitonic_sort_desc(sel, len);
            for (int i = tid; i < k; i += nthr) emit(i, (uint32_t)(sel[i] >> 32), topk_token(sel[i]));
        }
    }
    cl_sync();  // no rank leaves while another may still touch its shared memory
}

template <int U>
static int launch_topk_instance(const TopkParams& p, int grid, size_t smem, void* stream) {
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, topk_kernel<U>);
    if (e != cudaSuccess) return (int)e;
    if (fa.maxDynamicSharedSizeBytes < (int)smem) {
        e = cudaFuncSetAttribute(topk_kernel<U>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smem);
        if (e != cudaSuccess) return (int)e;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kTopkThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = static_cast<cudaStream_t>(stream);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return (int)cudaLaunchKernelEx(&cfg, topk_kernel<U>, p);
}

// Row mode, split over clusters of C CTAs (see topk_cluster_kernel).
static int launch_topk_cluster(const TopkParams& p, int rows, int C, size_t smem, void* stream) {
    auto kernel = topk_cluster_kernel<kTopkUnrollShort>;
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, kernel);
    if (e != cudaSuccess) return (int)e;
    if (fa.maxDynamicSharedSizeBytes < (int)smem) {
        e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return (int)e;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(rows * C));
    cfg.blockDim = dim3(kTopkThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = static_cast<cudaStream_t>(stream);
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return (int)cudaLaunchKernelEx(&cfg, kernel, p);
}

// Cluster size for row mode: rows that leave SMs idle (two CTAs per SM of the
// cluster kernel, 148 SMs) and are long enough to be worth splitting get 2
// CTAs each (4 measured no faster by token and slower by value: rank 0's
// gather and sort grow with the ranks); `force` (2 or 4; 1 = never)
// overrides the choice.
static int topk_cluster_size(int rows, int L, int force) {
    if (force == 1) return 1;
    if (force == 2 || force == kTopkMaxCluster) return force;
    if (L < kTopkClusterMinRow) return 1;
    if (rows * 2 <= 2 * kTopkSms) return 2;
    return 1;
}

// Long rows (row mode with L > kTopkLongRow) take the deeper-unrolled
// instance; merge mode reads no row from global memory after compaction.
static int launch_topk_params(const TopkParams& p, int grid, void* stream, int cluster = 1) {
    int sort_n = kTopkMinSort;
    while (sort_n < p.k) sort_n <<= 1;
    const size_t smem = (size_t)sort_n * 8 + (size_t)p.region_words * 4;
    if (p.shards == 0 && cluster > 1) return launch_topk_cluster(p, grid, cluster, smem, stream);
    if (p.shards == 0 && p.L > kTopkLongRow)
        return launch_topk_instance<kTopkUnrollLong>(p, grid, smem, stream);
    return launch_topk_instance<kTopkUnrollShort>(p, grid, smem, stream);
}

// Host launcher, row mode: one CTA per row. Shared memory: the sort buffer
// (next power of two >= k, at least 64 entries of 8 bytes) and a region of
// min(L rounded up to 4, 16384) words for cached keys or candidates.
// Launched with programmatic dependent launch, so it may start while the
// logits kernel before it drains.
int launch_topk(const float* logits, const int32_t* context_lens, int batch, int next_n, int L,
                int k, int flags, int32_t* out, float* values, void* stream, int cluster_force) {
    TopkParams p = {};
    p.logits = logits;
    p.context_lens = context_lens;
    p.out = out;
    p.values = values;
    p.next_n = next_n;
    p.L = L;
    p.k = k;
    const int L4 = (L + 3) & ~3;
    p.region_words = L4 < kTopkCacheKeys ? L4 : kTopkCacheKeys;
    p.by_token = (flags & MQA_TOPK_BY_TOKEN) ? 1 : 0;
    const int rows = batch * next_n;
    return launch_topk_params(p, rows, stream, topk_cluster_size(rows, L, cluster_force));
}

// Host launcher, merge mode: one CTA per row; the region holds all
// shards * k_in entries of a row as 8-byte candidates.
int launch_topk_merge(const float* cand_values, const int32_t* cand_tokens, int shards, int rows,
                      int k_in, const int32_t* offsets, int k, int flags, int32_t* out,
                      float* values, void* stream) {
    TopkParams p = {};
    p.logits = cand_values;
    p.cand_tokens = cand_tokens;
    p.out = out;
    p.values = values;
    p.k = k;
    p.rows = rows;
    p.shards = shards;
    p.k_in = k_in;
    for (int s = 0; s < shards; ++s) p.offsets[s] = offsets[s];
    p.region_words = 2 * shards * k_in;
    p.by_token = (flags & MQA_TOPK_BY_TOKEN) ? 1 : 0;
    return launch_topk_params(p, rows, stream);
}

}  // namespace mqa
