// topk.cu -- exact arg-top-K of a score row (Sec. 2.2 Eq. 2; Sec. 3.1 S_sparse; Sec. 3.3
// page top-M and Eq. 11), as a radix select on the order-preserving 32-bit key of each score.
//
// Ranking: (score desc, slot asc); slots are in position order, so ties go to the lower
// position.  Output: the selected positions sorted ascending, -1 in unused slots.
//
// Calls of up to kSmallRowsMax rows of at most kSmallMax slots take one launch
// (select_small_kernel, below).  Others take three launches per call, all rows at once:
//   hist    : per (row, chunk) CTA, a shared-memory histogram of the top 12 key bits,
//             flushed into the row's global histogram;
//   collect : every CTA of a row derives the same threshold digit from the row histogram,
//             then appends slots above it to the row's "sure" list (fewer than K of them)
//             and slots equal to it to the "candidate" list (warp-aggregated atomics);
//   final   : one CTA per row resolves the remaining 20 key bits among the candidates
//             (two more digit passes), breaks exact-key ties by the lowest slots (a radix
//             select on slot bits), then bitonic-sorts the K winners and writes positions.
// The histogram of the first digit is what makes the candidate list short: for score rows
// of the workloads here it holds ~1-2% of the row.  Any distribution, including all-equal
// scores, still gives the exact answer (the candidate list then holds the whole row).
#include "lsa_internal.cuh"
#include "select_util.cuh"

namespace lsa {
namespace {

constexpr int kThreads = 512;
constexpr int kFinalThreads = 1024;
constexpr int64_t kChunk = 16384;
constexpr int kCandCache = 8192;  // candidates cached in shared memory by the final pass

__global__ void __launch_bounds__(kThreads) select_hist_kernel(SelectArgs a, int64_t row0) {
    __shared__ uint32_t h[kHistBins];
    const int64_t r = row0 + blockIdx.y;
    int64_t lo, hi;
    if (!select_row_range(a, r, lo, hi)) return;
    const int64_t start = lo + (int64_t)blockIdx.x * kChunk;
    if (start >= hi) return;
    const int64_t end = min(hi, start + kChunk);
    for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) h[i] = 0;
    __syncthreads();
    const float *s = a.scores + r * a.row_stride;
    for (int64_t i = start + threadIdx.x; i < end; i += blockDim.x) {
        const uint32_t k = order_key(s[i]);
        if (k) atomicAdd(&h[k >> (32 - kHistBits)], 1u);
    }
    __syncthreads();
    uint32_t *gh = a.hist + r * kHistBins;
    for (int i = threadIdx.x; i < kHistBins; i += blockDim.x)
        if (h[i]) atomicAdd(&gh[i], h[i]);
}

// Collect pass: appends every key of the chunk above the threshold bin to the row's sure list and
// every key in it to the candidate list.  All of a thread's keys are loaded in one batch into
// registers; the CTA then takes its slots of both lists with a block-wide prefix count and one
// atomic per list, so no key waits on a round trip to global memory.
constexpr int kVecPerThread = (int)(kChunk / 4 / kThreads);  // 8 float4 per thread
static_assert(kChunk % (4 * kThreads) == 0, "chunk must be whole float4 rounds");

__global__ void __launch_bounds__(kThreads) select_collect_kernel(SelectArgs a, int64_t row0) {
    __shared__ uint32_t h[kHistBins];
    __shared__ uint32_t scratch[40];
    __shared__ uint32_t wsum[kThreads / 32];
    __shared__ int base_s[2];
    const int64_t r = row0 + blockIdx.y;
    int64_t lo, hi;
    if (!select_row_range(a, r, lo, hi)) return;
    const int64_t start = lo + (int64_t)blockIdx.x * kChunk;
    if (start >= hi) return;
    const int64_t end = min(hi, start + kChunk);
    int32_t *cnt = a.counts + r * kCountStride;
    int thr;
    if (a.thr_ready) {
        // the scorer's last CTA of this row already derived the threshold digit
        thr = cnt[2];
    } else {
        const uint32_t *gh = a.hist + r * kHistBins;
        for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) h[i] = gh[i];
        __syncthreads();
        uint32_t gt, total;
        row_threshold(h, a.K, &thr, &gt, &total, scratch);
        if (blockIdx.x == 0 && threadIdx.x == 0) {
            cnt[2] = thr;
            cnt[3] = (int32_t)total;
        }
    }
    const float *sc = a.scores + r * a.row_stride;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // [start, end) = scalar head up to the first 16-byte boundary (threads 0-2), float4 body,
    // scalar tail (threads 3-5); only elements of the range are read
    const int64_t n = end - start;
    const int64_t head =
        min(n, (int64_t)((4 - ((reinterpret_cast<uintptr_t>(sc + start) >> 2) & 3)) & 3));
    const int64_t n4 = (n - head) >> 2;
    const int64_t tail0 = start + head + 4 * n4;
    const float4 *v4 = reinterpret_cast<const float4 *>(sc + start + head);
    uint32_t k[kVecPerThread][4];
#pragma unroll
    for (int u = 0; u < kVecPerThread; ++u) {
        const int64_t j = (int64_t)u * kThreads + tid;
        const float4 x = j < n4 ? v4[j] : make_float4(0.f, 0.f, 0.f, 0.f);
        const bool in = j < n4;
        k[u][0] = in ? order_key(x.x) : 0u;
        k[u][1] = in ? order_key(x.y) : 0u;
        k[u][2] = in ? order_key(x.z) : 0u;
        k[u][3] = in ? order_key(x.w) : 0u;
    }
    int64_t xi = -1;  // this thread's scalar element (head or tail), if any
    if (tid < 3) {
        if (tid < head) xi = start + tid;
    } else if (tid < 6) {
        if (tail0 + (tid - 3) < end) xi = tail0 + (tid - 3);
    }
    const uint32_t xk = xi >= 0 ? order_key(sc[xi]) : 0u;
    auto is_sure = [&](uint32_t key) { return key != 0 && (int)(key >> (32 - kHistBits)) > thr; };
    auto is_cand = [&](uint32_t key) { return key != 0 && (int)(key >> (32 - kHistBits)) == thr; };
    // counts packed as sure (low 16 bits) + cand (high 16 bits); a CTA holds at most 16384 keys
    uint32_t c = (uint32_t)is_sure(xk) | ((uint32_t)is_cand(xk) << 16);
#pragma unroll
    for (int u = 0; u < kVecPerThread; ++u)
#pragma unroll
        for (int e = 0; e < 4; ++e) c += (uint32_t)is_sure(k[u][e]) | ((uint32_t)is_cand(k[u][e]) << 16);
    // block exclusive prefix of c
    uint32_t incl = c;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const uint32_t v = __shfl_up_sync(0xFFFFFFFFu, incl, d);
        if (lane >= d) incl += v;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const uint32_t v = lane < kThreads / 32 ? wsum[lane] : 0u;
        uint32_t wi = v;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const uint32_t u = __shfl_up_sync(0xFFFFFFFFu, wi, d);
            if (lane >= d) wi += u;
        }
        if (lane < kThreads / 32) wsum[lane] = wi - v;  // exclusive over warps
        if (lane == kThreads / 32 - 1) {
            // this CTA's slots in both lists (the counters may run past the lists' capacity;
            // the final pass never reads beyond what fits)
            base_s[0] = (wi & 0xFFFFu) ? atomicAdd(&cnt[0], (int)(wi & 0xFFFFu)) : 0;
            base_s[1] = (wi >> 16) ? atomicAdd(&cnt[1], (int)(wi >> 16)) : 0;
        }
    }
    __syncthreads();
    const uint32_t ex = wsum[warp] + incl - c;
    int ps = base_s[0] + (int)(ex & 0xFFFFu);
    int64_t pc = (int64_t)base_s[1] + (ex >> 16);
    auto put = [&](uint32_t key, int64_t i) {
        if (is_sure(key)) {
            if (ps < a.sure_stride) a.sure[r * a.sure_stride + ps] = (int32_t)i;
            else raise_error(a.err, LSA_DEVERR_INTERNAL);
            ++ps;
        } else if (is_cand(key)) {
            if (pc < a.cand_stride) a.cand[r * a.cand_stride + pc] = (int32_t)i;
            else raise_error(a.err, LSA_DEVERR_INTERNAL);
            ++pc;
        }
    };
    if (c != 0) {
        put(xk, xi);
#pragma unroll
        for (int u = 0; u < kVecPerThread; ++u) {
            const int64_t i = start + head + 4 * ((int64_t)u * kThreads + tid);
#pragma unroll
            for (int e = 0; e < 4; ++e) put(k[u][e], i + e);
        }
    }
}

// Sort x (one value per thread, N <= blockDim = 1024, N a power of two, threads >= N hold
// INT32_MAX) ascending: bitonic network, partner distances < 32 by warp shuffles, larger ones
// through shared memory (xchg: blockDim words).
__device__ __forceinline__ int32_t bitonic_sort_1024(int32_t x, int N, int32_t *xchg) {
    const int t = threadIdx.x;
    for (int k = 2; k <= N; k <<= 1) {
        for (int j = k >> 1; j > 0; j >>= 1) {
            int32_t y;
            if (j >= 32) {
                xchg[t] = x;
                __syncthreads();
                y = xchg[t ^ j];
                __syncthreads();
            } else {
                y = __shfl_xor_sync(0xFFFFFFFFu, x, j);
            }
            const bool up = (t & k) == 0;
            const bool lower = (t & j) == 0;
            x = (lower == up) ? min(x, y) : max(x, y);
        }
    }
    return x;
}

__global__ void __launch_bounds__(kFinalThreads) select_final_kernel(SelectArgs a, int64_t row0) {
    extern __shared__ __align__(16) uint32_t fsm[];
    uint32_t *h = fsm;                                                // kHistBins
    int32_t *sel = reinterpret_cast<int32_t *>(fsm + kHistBins);      // kMaxSelect
    uint32_t *ckey = fsm + kHistBins + kMaxSelect;                    // kCandCache
    int32_t *cslot = reinterpret_cast<int32_t *>(ckey + kCandCache);  // kCandCache
    __shared__ uint32_t scratch[40];
    __shared__ int n_sel;
    const int64_t r = row0 + blockIdx.x;
    const int tid = threadIdx.x;
    int32_t *out = a.out + r * a.out_stride;
    int64_t lo, hi;
    if (!select_row_range(a, r, lo, hi)) {
        for (int i = tid; i < a.K; i += blockDim.x) out[i] = -1;
        if (a.out_count && tid == 0) a.out_count[r] = 0;
        return;
    }
    const int32_t *cnt = a.counts + r * kCountStride;
    // the counters keep counting past a full list (that case is flagged by collect); never
    // read beyond what was stored
    const int n_sure = min(cnt[0], a.sure_stride);
    const int n_cand = (int)min((int64_t)cnt[1], a.cand_stride);
    const int thr = cnt[2];
    const int total = cnt[3];
    const int K = a.K;
    const int K_eff = total < K ? total : K;
    const float *s = a.scores + r * a.row_stride;
    const int32_t *cand = a.cand + r * a.cand_stride;
    const bool cached = n_cand <= kCandCache;

    if (tid == 0) n_sel = min(n_sure, kMaxSelect);
    for (int i = tid; i < n_sure && i < kMaxSelect; i += blockDim.x) sel[i] = a.sure[r * a.sure_stride + i];
    if (cached) {
        for (int i = tid; i < n_cand; i += blockDim.x) {
            const int32_t sl = cand[i];
            cslot[i] = sl;
            ckey[i] = order_key(s[sl]);
        }
    }
    __syncthreads();
    auto key_of = [&](int i) -> uint32_t { return cached ? ckey[i] : order_key(s[cand[i]]); };
    auto slot_of = [&](int i) -> int32_t { return cached ? cslot[i] : cand[i]; };

    if (thr >= 0 && n_cand > 0) {
        const uint32_t need = (uint32_t)(K - n_sure);
        // digit 2: key bits [19:8]
        for (int i = tid; i < kHistBins; i += blockDim.x) h[i] = 0;
        __syncthreads();
        for (int i = tid; i < n_cand; i += blockDim.x) atomicAdd(&h[(key_of(i) >> 8) & 0xFFFu], 1u);
        __syncthreads();
        int d2;
        uint32_t gt2;
        find_threshold(h, 4096, need, &d2, &gt2, scratch);
        const uint32_t need2 = need - gt2;
        // digit 3: key bits [7:0] among the candidates of digit 2
        for (int i = tid; i < 256; i += blockDim.x) h[i] = 0;
        __syncthreads();
        for (int i = tid; i < n_cand; i += blockDim.x) {
            const uint32_t k = key_of(i);
            if ((int)((k >> 8) & 0xFFFu) == d2) atomicAdd(&h[k & 0xFFu], 1u);
        }
        __syncthreads();
        int d3;
        uint32_t gt3;
        find_threshold(h, 256, need2, &d3, &gt3, scratch);
        const uint32_t need_eq = need2 - gt3;
        const uint32_t eq_count = h[d3];
        __syncthreads();
        const uint32_t V = ((uint32_t)thr << 20) | ((uint32_t)d2 << 8) | (uint32_t)d3;
        int64_t slot_cut = 0x7FFFFFFFFFFFFFFFll;
        if (need_eq < eq_count) {
            // the need_eq lowest slots among candidates with key == V: radix select on the
            // slot value, smallest first (bins mirrored so "largest bin" = smallest digit)
            const int shifts[3] = {20, 10, 0};
            const int bits[3] = {11, 10, 10};
            uint32_t prefix = 0, need_s = need_eq;
            for (int dgt = 0; dgt < 3; ++dgt) {
                const int nb = 1 << bits[dgt], sh = shifts[dgt];
                for (int i = tid; i < nb; i += blockDim.x) h[i] = 0;
                __syncthreads();
                for (int i = tid; i < n_cand; i += blockDim.x) {
                    if (key_of(i) != V) continue;
                    const uint32_t slot = (uint32_t)slot_of(i);
                    if ((slot >> (sh + bits[dgt])) != prefix) continue;
                    atomicAdd(&h[nb - 1 - ((slot >> sh) & (nb - 1))], 1u);
                }
                __syncthreads();
                int fb;
                uint32_t gtb;
                find_threshold(h, nb, need_s, &fb, &gtb, scratch);
                need_s -= gtb;
                prefix = (prefix << bits[dgt]) | (uint32_t)(nb - 1 - fb);
            }
            slot_cut = prefix;
        }
        for (int i = tid; i < n_cand; i += blockDim.x) {
            const uint32_t k = key_of(i);
            const int32_t slot = slot_of(i);
            if (k > V || (k == V && (int64_t)slot <= slot_cut)) {
                const int p = atomicAdd(&n_sel, 1);
                if (p < kMaxSelect) sel[p] = slot;
            }
        }
    }
    __syncthreads();
    const int ns = n_sel;
    if (ns != K_eff && tid == 0) raise_error(a.err, LSA_DEVERR_INTERNAL);
    const int m = min(ns, min(K_eff, kMaxSelect));
    if (hi - lo <= (int64_t)kHistBins * 32) {
        // Ascending order without a sort: mark the selected slots in a bitmap over [lo, hi)
        // (the histogram buffer, 4 words per thread), count the marks of each thread's words,
        // and let every thread write its slots at its exclusive prefix count.
        for (int i = tid; i < kHistBins; i += blockDim.x) h[i] = 0u;
        __syncthreads();
        for (int i = tid; i < m; i += blockDim.x) {
            const int64_t d = (int64_t)sel[i] - lo;
            if (d >= 0 && d < hi - lo) atomicOr(&h[d >> 5], 1u << (d & 31));
            else raise_error(a.err, LSA_DEVERR_INTERNAL);
        }
        __syncthreads();
        constexpr int kWords = kHistBins / kFinalThreads;  // 4
        uint32_t w[kWords];
        int c = 0;
#pragma unroll
        for (int k = 0; k < kWords; ++k) {
            w[k] = h[tid * kWords + k];
            c += __popc(w[k]);
        }
        // block exclusive scan of c (warp shuffles, then the 32 warp totals)
        const int lane = tid & 31, warp = tid >> 5;
        int incl = c;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const int v = __shfl_up_sync(0xFFFFFFFFu, incl, d);
            if (lane >= d) incl += v;
        }
        if (lane == 31) scratch[warp] = (uint32_t)incl;
        __syncthreads();
        if (warp == 0) {
            int v = (int)scratch[lane], wi = v;
#pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                const int u = __shfl_up_sync(0xFFFFFFFFu, wi, d);
                if (lane >= d) wi += u;
            }
            scratch[lane] = (uint32_t)(wi - v);  // exclusive over warps
        }
        __syncthreads();
        int o = (int)scratch[warp] + incl - c;
#pragma unroll
        for (int k = 0; k < kWords; ++k) {
            uint32_t x = w[k];
            while (x) {
                const int bit = __ffs(x) - 1;
                x &= x - 1;
                if (o < K)
                    out[o] = (int32_t)slot_to_pos(a, r, lo + (int64_t)(tid * kWords + k) * 32 + bit);
                ++o;
            }
        }
        for (int i = m + tid; i < K; i += blockDim.x) out[i] = -1;
        if (a.out_count && tid == 0) a.out_count[r] = m;
        return;
    }
    int N = 2;
    while (N < m) N <<= 1;
    if (N <= (int)blockDim.x) {
        int32_t x = (tid < m) ? sel[tid] : 0x7FFFFFFF;
        __syncthreads();
        x = bitonic_sort_1024(x, N, sel);
        if (tid < m) sel[tid] = x;
        __syncthreads();
    } else {
        // K > 1024: plain shared-memory bitonic network over N = 2048 or 4096 entries
        for (int i = m + tid; i < N; i += blockDim.x) sel[i] = 0x7FFFFFFF;
        __syncthreads();
        for (int k = 2; k <= N; k <<= 1) {
            for (int j = k >> 1; j > 0; j >>= 1) {
                for (int i = tid; i < N; i += blockDim.x) {
                    const int ixj = i ^ j;
                    if (ixj > i) {
                        const int32_t x = sel[i], y = sel[ixj];
                        const bool up = (i & k) == 0;
                        if ((x > y) == up) {
                            sel[i] = y;
                            sel[ixj] = x;
                        }
                    }
                }
                __syncthreads();
            }
        }
    }
    for (int i = tid; i < K; i += blockDim.x)
        out[i] = (i < m) ? (int32_t)slot_to_pos(a, r, sel[i]) : -1;
    if (a.out_count && tid == 0) a.out_count[r] = m;
}

// ---------------------------------------------------------------- rows of few slots
// One CTA (1024 threads) per row holds the row's keys in shared memory and resolves the whole
// selection in one launch: the three digit passes (bits 31:20, 19:8, 7:0) find the key V of the
// K-th largest entry; warp ballots then build bitmaps of the slots above V and equal to V, one
// block scan keeps the lowest equal slots (ties go to the lower position), and a second gives
// every selected slot its place in the ascending output.  Same result as collect + final.
constexpr int kSmallMax = 16384;               // slots per row the one-launch select takes
constexpr int kSmallWords = kSmallMax / 32;    // bitmap words
constexpr int kSmallThreads = 1024;
constexpr int kSmallSmem = (kSmallMax + kHistBins + 2 * kSmallWords) * 4;
constexpr int64_t kSmallRowsMax = 512;         // rows per call the one-launch select takes

// Exclusive block scan of one value per thread (1024 threads); every thread gets its prefix
// and the total.
__device__ __forceinline__ uint32_t block_exclusive_scan(uint32_t v, uint32_t *scratch,
                                                         uint32_t *total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t incl = v;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const uint32_t u = __shfl_up_sync(0xFFFFFFFFu, incl, d);
        if (lane >= d) incl += u;
    }
    if (lane == 31) scratch[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const uint32_t wv = scratch[lane];
        uint32_t wi = wv;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const uint32_t u = __shfl_up_sync(0xFFFFFFFFu, wi, d);
            if (lane >= d) wi += u;
        }
        scratch[lane] = wi - wv;  // exclusive over warps
        if (lane == 31) scratch[32] = wi;
    }
    __syncthreads();
    const uint32_t ex = scratch[warp] + incl - v;
    *total = scratch[32];
    __syncthreads();
    return ex;
}

__global__ void __launch_bounds__(kSmallThreads) select_small_kernel(SelectArgs a, int64_t row0) {
    extern __shared__ __align__(16) uint32_t ssm[];
    uint32_t *key = ssm;                       // [kSmallMax]
    uint32_t *h = ssm + kSmallMax;             // [kHistBins]
    uint32_t *gtmap = h + kHistBins;           // [kSmallWords]
    uint32_t *eqmap = gtmap + kSmallWords;     // [kSmallWords]
    __shared__ uint32_t scratch[40];
    const int64_t r = row0 + blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31;
    int32_t *out = a.out + r * a.out_stride;
    const int K = a.K;
    int64_t lo, hi;
    if (!select_row_range(a, r, lo, hi) || hi - lo > kSmallMax) {
        if (hi - lo > kSmallMax && tid == 0) raise_error(a.err, LSA_DEVERR_INTERNAL);
        for (int i = tid; i < K; i += blockDim.x) out[i] = -1;
        if (a.out_count && tid == 0) a.out_count[r] = 0;
        return;
    }
    const int n = (int)(hi - lo);
    const int nw = (n + 31) >> 5;
    const float *s = a.scores + r * a.row_stride + lo;
    uint32_t c = 0;
    for (int i = tid; i < n; i += blockDim.x) {
        const uint32_t k = order_key(s[i]);  // 0: excluded slot
        key[i] = k;
        c += (k != 0);
    }
    const uint32_t total = block_sum(c, scratch);  // its barrier also publishes key[]
    const uint32_t K_eff = total < (uint32_t)K ? total : (uint32_t)K;
    uint32_t V = 0, need_eq = 0;  // total <= K: every non-excluded slot (key > 0) is taken
    if (total > (uint32_t)K) {
        // digit 1: bits 31:20
        for (int i = tid; i < kHistBins; i += blockDim.x) h[i] = 0;
        __syncthreads();
        for (int i = tid; i < n; i += blockDim.x) {
            const uint32_t k = key[i];
            if (k) atomicAdd(&h[k >> 20], 1u);
        }
        __syncthreads();
        int d1, d2, d3;
        uint32_t gt1, gt2, gt3;
        find_threshold(h, kHistBins, (uint32_t)K, &d1, &gt1, scratch);
        // digit 2: bits 19:8 among keys with digit 1 = d1
        for (int i = tid; i < kHistBins; i += blockDim.x) h[i] = 0;
        __syncthreads();
        for (int i = tid; i < n; i += blockDim.x) {
            const uint32_t k = key[i];
            if (k && (int)(k >> 20) == d1) atomicAdd(&h[(k >> 8) & 0xFFFu], 1u);
        }
        __syncthreads();
        const uint32_t need1 = (uint32_t)K - gt1;
        find_threshold(h, kHistBins, need1, &d2, &gt2, scratch);
        // digit 3: bits 7:0 among keys with digits 1, 2 = d1, d2
        const uint32_t hi24 = ((uint32_t)d1 << 12) | (uint32_t)d2;
        for (int i = tid; i < 256; i += blockDim.x) h[i] = 0;
        __syncthreads();
        for (int i = tid; i < n; i += blockDim.x) {
            const uint32_t k = key[i];
            if (k && (k >> 8) == hi24) atomicAdd(&h[k & 0xFFu], 1u);
        }
        __syncthreads();
        const uint32_t need2 = need1 - gt2;
        find_threshold(h, 256, need2, &d3, &gt3, scratch);
        V = (hi24 << 8) | (uint32_t)d3;
        need_eq = need2 - gt3;
    }
    // bitmaps of the slots above V and equal to V (one warp ballot per 32 slots)
    for (int base = 0; base < nw * 32; base += blockDim.x) {
        const int i = base + tid;
        const uint32_t k = i < n ? key[i] : 0u;
        const uint32_t g = __ballot_sync(0xFFFFFFFFu, k > V);
        const uint32_t e = __ballot_sync(0xFFFFFFFFu, V != 0 && k == V);
        if (lane == 0 && (i >> 5) < nw) {
            gtmap[i >> 5] = g;
            eqmap[i >> 5] = e;
        }
    }
    __syncthreads();
    // thread t owns bitmap word t (nw <= kSmallWords <= blockDim.x): the lowest need_eq equal
    // slots across the row, then every selected slot's place in the output
    const uint32_t ew = tid < nw ? eqmap[tid] : 0u;
    uint32_t n_eq;
    const uint32_t eq_before = block_exclusive_scan((uint32_t)__popc(ew), scratch, &n_eq);
    uint32_t take = 0;  // the lowest (need_eq - eq_before) set bits of ew
    if (eq_before < need_eq) {
        uint32_t room = need_eq - eq_before;
        for (uint32_t x = ew; x && room; --room) {
            const uint32_t low = x & (0u - x);
            take |= low;
            x ^= low;
        }
    }
    const uint32_t sw = (tid < nw ? gtmap[tid] : 0u) | take;
    uint32_t m;
    uint32_t o = block_exclusive_scan((uint32_t)__popc(sw), scratch, &m);
    for (uint32_t x = sw; x; x &= x - 1) {
        const int bit = __ffs(x) - 1;
        if (o < (uint32_t)K) out[o] = (int32_t)slot_to_pos(a, r, lo + (int64_t)tid * 32 + bit);
        ++o;
    }
    if (m != K_eff && tid == 0) raise_error(a.err, LSA_DEVERR_INTERNAL);
    for (int i = (int)m + tid; i < K; i += blockDim.x) out[i] = -1;
    if (a.out_count && tid == 0) a.out_count[r] = (int32_t)m;
}

}  // namespace

bool select_is_small(int64_t rows, int64_t max_slots) {
    return max_slots <= kSmallMax && rows <= kSmallRowsMax;
}

cudaError_t select_clear(const SelectArgs &a, int64_t rows, cudaStream_t s) {
    cudaError_t e = cudaMemsetAsync(a.hist, 0, (size_t)rows * kHistBins * sizeof(uint32_t), s);
    if (e != cudaSuccess) return e;
    return cudaMemsetAsync(a.counts, 0, (size_t)rows * kCountStride * sizeof(int32_t), s);
}

cudaError_t launch_select(const SelectArgs &a, int64_t rows, int64_t max_slots, cudaStream_t s,
                          bool hist_ready) {
    if (rows <= 0) return cudaSuccess;
    cudaError_t e;
    if (select_is_small(rows, max_slots)) {
        // short rows: the whole selection in one launch, one CTA per row (many rows go to the
        // collect + final passes, which spread a row over several CTAs)
        if ((e = cudaFuncSetAttribute(select_small_kernel,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      kSmallSmem)) != cudaSuccess)
            return e;
        for (int64_t r0 = 0; r0 < rows; r0 += 0x7FFFFFFF) {
            const int64_t nr = rows - r0 < 0x7FFFFFFF ? rows - r0 : 0x7FFFFFFF;
            select_small_kernel<<<(unsigned)nr, kSmallThreads, kSmallSmem, s>>>(a, r0);
            if ((e = launched()) != cudaSuccess) return e;
        }
        return cudaSuccess;
    }
    if (!hist_ready && (e = select_clear(a, rows, s)) != cudaSuccess) return e;
    const int64_t chunks = max_slots > 0 ? (max_slots + kChunk - 1) / kChunk : 0;
    for (int64_t r0 = 0; r0 < rows; r0 += 65535) {
        const int64_t nr = rows - r0 < 65535 ? rows - r0 : 65535;
        if (chunks > 0) {
            dim3 grid((unsigned)chunks, (unsigned)nr);
            if (!hist_ready) {
                select_hist_kernel<<<grid, kThreads, 0, s>>>(a, r0);
                if ((e = launched()) != cudaSuccess) return e;
            }
            select_collect_kernel<<<grid, kThreads, 0, s>>>(a, r0);
            if ((e = launched()) != cudaSuccess) return e;
        }
    }
    const int fsmem = (kHistBins + kMaxSelect + 2 * kCandCache) * 4;
    if ((e = cudaFuncSetAttribute(select_final_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  fsmem)) != cudaSuccess)
        return e;
    for (int64_t r0 = 0; r0 < rows; r0 += 0x7FFFFFFF) {
        const int64_t nr = rows - r0 < 0x7FFFFFFF ? rows - r0 : 0x7FFFFFFF;
        select_final_kernel<<<(unsigned)nr, kFinalThreads, fsmem, s>>>(a, r0);
        if ((e = launched()) != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace lsa
