// attend_tc.cu -- Hybrid Sparse Attention forward on the 5th-generation tensor cores.
//
// Paper: Sec. 2.2 (u_t = Attn over the MLA latent rows c_s of S_t), Sec. 3.1 (S_t = sink U swa U
// S_sparse; the fixed tokens take part in the same softmax, Fig. 1), Sec. 4.1.1 (HFA: the
// contiguous and gathered branches merged by online-softmax rescaling).
//
// One query's work is two matrix products with the 128 heads as the MMA's M = 128 rows:
//   S = Q K^T   (N = 16 keys per tile, K = 576 latent dims)      -> TMEM, 16 columns
//   O += P V    (N = 256 value dims, K = 16 keys)                -> TMEM, 256 columns
// A 128 x 512 fp32 O would fill all of TMEM, so each CTA of a pair owns half of the value dims
// (blockIdx.y) and both recompute S; the key rows are read from HBM once and from L2 by the twin.
// Key/value rows are gathered by TMA tile::gather4 into the SWIZZLE_128B K-major layout (nine
// 64-dim chunks of 16 rows); the same tile is the B operand of S (K-major) and, read MN-major,
// of P V -- no transpose.  P goes through shared memory (K-major, no swizzle).
// Softmax is thread-per-head straight out of TMEM.  O is rescaled lazily: only when a head's
// running max grows by more than 2^8 is O read back, scaled and stored (after the previous P V
// has completed); otherwise P is formed against the stale max, which is exact.
//
// Warp roles (192 threads): warps 0-3 softmax + epilogue (thread = head = TMEM lane),
// warp 4 producer (position lookup, index validation, TMA gather into a ring of 4 stages),
// warp 5 TMEM allocator + single-thread MMA issuer.  Every wait is bounded (LSA_DEVERR_TIMEOUT).
//
// Grid: (query rows, 2 value halves, key splits); splits are merged by hfa_combine_kernel.
#include "lsa_internal.cuh"
#include "score_tc.cuh"
#include "tc_ptx.cuh"

namespace lsa {
namespace {

using namespace tc;

constexpr int DQK = 576;
constexpr int NCH = 9;     // 64-dim chunks of a latent row
constexpr int NK = 16;     // keys per tile
constexpr int STAGES = 4;
constexpr int HEADS = 128;
constexpr int DVH = 256;   // value dims per CTA
constexpr int kThreads = 192;
constexpr float kRescaleLog2 = 8.f;

constexpr int kQBytes = NCH * HEADS * 128;       // 147456
constexpr int kChunkBytes = NK * 128;            // 2048
constexpr int kStageBytes = NCH * kChunkBytes;   // 18432
constexpr int kPBytes = HEADS * NK * 2;          // 4096 (one P buffer)
constexpr int OFF_Q = 0;
constexpr int OFF_KV = OFF_Q + kQBytes;
constexpr int OFF_P = OFF_KV + STAGES * kStageBytes;
constexpr int OFF_OK = OFF_P + kPBytes;
constexpr int OFF_BAR = OFF_OK + STAGES * NK * 4;
constexpr int kNumBars = 2 * STAGES + 2 + 2 + 2 + 2 + 1;
constexpr int OFF_MISC = OFF_BAR + kNumBars * 8;
constexpr int kSmem = OFF_MISC + 16;
constexpr int kSmemLaunch = kSmem + 1024;        // slack to align the base to 1024
static_assert(kSmemLaunch <= 232448, "shared memory plan exceeds 227 KB");

struct RowKeys {
    int64_t n_sink, n_swa, swa_lo, n_sp, dyn_lo, dyn_hi;
    const int32_t *idx;
};

// Position of virtual key v (sink | window | gathered), -1 if none or invalid.
__device__ __forceinline__ int64_t key_pos(const RowKeys &L, int64_t v, bool check, int32_t *err) {
    if (v < L.n_sink) return v;
    v -= L.n_sink;
    if (v < L.n_swa) return L.swa_lo + v;
    v -= L.n_swa;
    if (v >= L.n_sp) return -1;
    const int64_t p = L.idx[v];
    const bool ok = p >= L.dyn_lo && p < L.dyn_hi && (v == 0 || L.idx[v - 1] < p);
    if (!ok) {
        if (check) raise_error(err, LSA_DEVERR_INDEX);
        return -1;
    }
    return p;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

__global__ void __launch_bounds__(kThreads, 1) hfa_tc_kernel(const __grid_constant__ CUtensorMap cmap,
                                                        AttendArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
    uint8_t *q_s = sm + OFF_Q;
    uint8_t *kv_s = sm + OFF_KV;
    uint8_t *p_s = sm + OFF_P;
    int *tile_ok = reinterpret_cast<int *>(sm + OFF_OK);
    uint64_t *full = reinterpret_cast<uint64_t *>(sm + OFF_BAR);
    uint64_t *empty = full + STAGES;
    uint64_t *sfull = empty + STAGES;
    uint64_t *sfree = sfull + 2;
    uint64_t *pfull = sfree + 2;
    uint64_t *pvdone = pfull + 2;
    uint64_t *drain = pvdone + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + OFF_MISC);
    volatile int *abort = reinterpret_cast<volatile int *>(sm + OFF_MISC + 4);
    int *nsp_s = reinterpret_cast<int *>(sm + OFF_MISC + 8);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t r = blockIdx.x;
    const int half = blockIdx.y;
    const int split = blockIdx.z;
    const int64_t b = r / a.T;
    const int64_t t = a.q_pos[r];
    const int64_t len = a.kv_len[b];
    if (!(t >= 0 && t < len && len <= a.L_max)) {
        if (tid == 0 && half == 0 && split == 0) raise_error(a.err, LSA_DEVERR_QPOS);
        return;
    }
    const Regions g = regions_of(t, a.Ks, a.Kw);
    RowKeys L;
    L.n_sink = g.sink_hi;
    L.n_swa = g.swa_hi - g.swa_lo;
    L.swa_lo = g.swa_lo;
    L.dyn_lo = g.dyn_lo;
    L.dyn_hi = g.dyn_hi;
    L.idx = a.idx + r * a.K;
    if (tid == 0) *nsp_s = 0;
    __syncthreads();
    {
        int c = 0;
        for (int i = tid; i < a.K; i += kThreads) c += (L.idx[i] >= 0);
        if (c) atomicAdd(nsp_s, c);
    }
    __syncthreads();
    L.n_sp = *nsp_s;
    const int64_t n_total = L.n_sink + L.n_swa + L.n_sp;
    const int64_t ntiles = (n_total + NK - 1) / NK;
    const int64_t t0 = (int64_t)split * a.tiles_per_split;
    int64_t t1 = t0 + a.tiles_per_split;
    if (t1 > ntiles) t1 = ntiles;
    const int n = (int)(t1 > t0 ? t1 - t0 : 0);
    const int H = a.H;  // == 128
    if (n == 0) {
        // an empty split: a zero partial with lse = -inf (only reachable with several splits)
        if (a.n_split > 1) {
            for (int i = tid; i < HEADS * DVH; i += kThreads) {
                const int h = i / DVH, d = i - h * DVH;
                a.part_o[((r * H + h) * a.n_split + split) * (int64_t)512 + half * DVH + d] = 0.f;
            }
            if (half == 0)
                for (int h = tid; h < HEADS; h += kThreads)
                    a.part_lse[(r * H + h) * a.n_split + split] = -INFINITY;
        }
        return;
    }

    // ---- set-up: Q (SWIZZLE_128B K-major, nine chunks), barriers, TMEM
    {
        // all 9216 16-byte pieces in flight at once (asynchronous copies), swizzled in place
        const __nv_bfloat16 *qr = a.q + r * (int64_t)H * DQK;
        for (int i = tid; i < HEADS * NCH * 8; i += kThreads) {
            const int h = i / (NCH * 8), rem = i - h * (NCH * 8), c = rem >> 3, p = rem & 7;
            cp_async16(q_s + c * (HEADS * 128) + h * 128 + ((p ^ (h & 7)) << 4),
                       qr + h * DQK + c * 64 + p * 8, 16);
        }
        cp_async_commit();
        if (tid == 0) {
            for (int s = 0; s < STAGES; ++s) {
                mbar_init(&full[s], 1);
                mbar_init(&empty[s], 1);
            }
            for (int s = 0; s < 2; ++s) {
                mbar_init(&sfull[s], 1);
                mbar_init(&sfree[s], 128);
                mbar_init(&pfull[s], 128);
                mbar_init(&pvdone[s], 1);
            }
            mbar_init(drain, 1);
            *abort = 0;
            asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        }
        if (warp == 5) {
            asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                         ::"r"(smem_u32(tmem_slot)), "r"(512));
            asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
        }
        cp_async_wait<0>();
        fence_proxy_async();
        fence_before();
        __syncthreads();
        fence_after();
    }
    const uint32_t tmem = *tmem_slot;

    if (warp == 4) {
        // ------------------------------------------------------------ producer (one warp)
        // Key rows are gathered by TMA tile::gather4: four rows x one 64-dim chunk (4 x 128 B,
        // swizzled in place) per instruction, 36 instructions per 16-row tile, completing the
        // stage's barrier by byte count.  Lane j < 16 owns row j: it looks its position up one
        // tile ahead and validates it; an invalid key reads a valid row and is masked later.
        const int64_t row_base = b * a.L_max;
        int64_t pos = (lane < NK) ? key_pos(L, t0 * NK + lane, true, a.err) : -1;
        int issued = 0;
        for (int i = 0; i < n; ++i) {
            const int s = i % STAGES;
            bool ok = true;
            if (i >= STAGES) ok = mbar_wait(&empty[s], ((i / STAGES) & 1) ^ 1, abort, a.err);
            if (!__all_sync(0xFFFFFFFFu, ok)) break;
            if (lane < NK) tile_ok[s * NK + lane] = (pos >= 0);
            const int rc = (int)(row_base + (pos >= 0 ? pos : 0));
            const int g = lane & 3;
            const int r0 = __shfl_sync(0xFFFFFFFFu, rc, 4 * g);
            const int r1 = __shfl_sync(0xFFFFFFFFu, rc, 4 * g + 1);
            const int r2 = __shfl_sync(0xFFFFFFFFu, rc, 4 * g + 2);
            const int r3 = __shfl_sync(0xFFFFFFFFu, rc, 4 * g + 3);
            __syncwarp();
            if (lane == 0) mbar_expect_tx(&full[s], kStageBytes);
            __syncwarp();
            uint8_t *base = kv_s + s * kStageBytes;
            // lane -> chunk lane/4 (0..7), row group lane%4; lanes 0-3 also take chunk 8
            tma_gather4(base + (lane >> 2) * kChunkBytes + g * 512, &cmap, (lane >> 2) * 64, r0,
                        r1, r2, r3, &full[s]);
            if (lane < 4)
                tma_gather4(base + 8 * kChunkBytes + g * 512, &cmap, 8 * 64, r0, r1, r2, r3,
                            &full[s]);
            ++issued;
            if (i + 1 < n) pos = (lane < NK) ? key_pos(L, (t0 + i + 1) * NK + lane, true, a.err) : -1;
        }
        if (*abort && lane == 0) {
            // let the copies already issued land before the CTA may exit
            for (int k = (issued > STAGES ? issued - STAGES : 0); k < issued; ++k) {
                const uint64_t ts = globaltimer();
                while (!mbar_try(&full[k % STAGES], (k / STAGES) & 1))
                    if (globaltimer() - ts > kWaitNs) break;
            }
        }
    } else if (warp == 5) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc_s = (1u << 4) | (1u << 7) | (1u << 10) |
                                     ((uint32_t)(NK >> 3) << 17) | ((uint32_t)(HEADS >> 4) << 24);
            const uint32_t idesc_pv = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) |
                                      ((uint32_t)(DVH >> 3) << 17) |
                                      ((uint32_t)(HEADS >> 4) << 24);
            const uint32_t q_addr = smem_u32(q_s), kv_addr = smem_u32(kv_s);
            const uint32_t p_addr = smem_u32(p_s);
            const uint32_t o_tmem = tmem + 256;
            bool live = true;
            auto issue_s = [&](int i) -> bool {
                const int s = i % STAGES, bb = i & 1;
                if (!mbar_wait(&full[s], (i / STAGES) & 1, abort, a.err)) return false;
                if (i >= 2 && !mbar_wait(&sfree[bb], ((i >> 1) & 1) ^ 1, abort, a.err))
                    return false;
                fence_after();
                const uint32_t kvb = kv_addr + s * kStageBytes;
#pragma unroll 4
                for (int kk = 0; kk < DQK / 16; ++kk) {
                    const int c = kk >> 2, o = (kk & 3) * 32;
                    const uint64_t ad = smem_desc(q_addr + c * (HEADS * 128) + o, 16, 1024, 2);
                    const uint64_t bd = smem_desc(kvb + c * kChunkBytes + o, 16, 1024, 2);
                    umma_bf16(tmem + bb * NK, ad, bd, idesc_s, kk > 0);
                }
                umma_commit(&sfull[bb]);
                return true;
            };
            live = issue_s(0);
            for (int i = 0; i < n && live; ++i) {
                if (i + 1 < n && !issue_s(i + 1)) break;
                if (!mbar_wait(&pfull[i & 1], (i >> 1) & 1, abort, a.err)) break;
                fence_after();
                const int s = i % STAGES;
                const uint64_t ad = smem_desc(p_addr, 128, 256, 0);
                const uint64_t bd =
                    smem_desc(kv_addr + s * kStageBytes + half * 4 * kChunkBytes, kChunkBytes, 1024,
                              2);
                umma_bf16(o_tmem, ad, bd, idesc_pv, i > 0);
                umma_commit(&empty[s]);
                umma_commit(&pvdone[i & 1]);
            }
            umma_commit(drain);
            const uint64_t ts = globaltimer();
            while (!mbar_try(drain, 0))
                if (globaltimer() - ts > kWaitNs) {
                    raise_error(a.err, LSA_DEVERR_TIMEOUT);
                    break;
                }
        }
    } else {
        // ------------------------------------------------------------ softmax + epilogue
        const int h = tid;  // head = TMEM lane
        const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
        const uint32_t o_tmem = tmem + lane_base + 256;
        float m_ref = -INFINITY, l = 0.f;
        bool nonfinite = false, live = true;
        for (int i = 0; i < n; ++i) {
            const int bb = i & 1, s = i % STAGES;
            bool ok = mbar_wait(&sfull[bb], (i >> 1) & 1, abort, a.err);
            ok = ok && mbar_wait(&full[s], (i / STAGES) & 1, abort, a.err);
            if (!__all_sync(0xFFFFFFFFu, ok)) {
                live = false;
                break;
            }
            fence_after();
            uint32_t v[NK];
            tmem_ld16(tmem + lane_base + bb * NK, v);
            tmem_wait_ld();
            fence_before();
            mbar_arrive(&sfree[bb]);
            float z[NK];
            float mt = -INFINITY;
#pragma unroll
            for (int j = 0; j < NK; ++j) {
                const float x = __uint_as_float(v[j]) * a.scale_log2;
                nonfinite |= !isfinite(x);
                z[j] = tile_ok[s * NK + j] ? x : -INFINITY;
                mt = fmaxf(mt, z[j]);
            }
            const bool need = (m_ref == -INFINITY) ? (mt > -INFINITY) : (mt > m_ref + kRescaleLog2);
            if (__any_sync(0xFFFFFFFFu, need)) {
                float alpha = 1.f, m_new = m_ref;
                if (need) {
                    m_new = fmaxf(m_ref, mt);
                    alpha = (m_ref == -INFINITY) ? 0.f : exp2f(m_ref - m_new);
                }
                if (i > 0) {
                    // O holds the P V of tiles < i: wait for the last one, then scale in place
                    const bool okp = mbar_wait(&pvdone[(i - 1) & 1], ((i - 1) >> 1) & 1, abort,
                                               a.err);
                    if (!__all_sync(0xFFFFFFFFu, okp)) {
                        live = false;
                        break;
                    }
                    fence_after();
#pragma unroll 1
                    for (int ch = 0; ch < DVH / 32; ++ch) {
                        uint32_t ov[32];
                        tmem_ld32(o_tmem + ch * 32, ov);
                        tmem_wait_ld();
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            ov[j] = __float_as_uint(__uint_as_float(ov[j]) * alpha);
                        tmem_st32(o_tmem + ch * 32, ov);
                    }
                    tmem_wait_st();
                    fence_before();
                }
                l *= alpha;
                m_ref = m_new;
            }
            float p[NK];
            float rs = 0.f;
#pragma unroll
            for (int j = 0; j < NK; ++j) {
                p[j] = (m_ref == -INFINITY) ? 0.f : exp2f(z[j] - m_ref);
                rs += p[j];
            }
            l += rs;
            if (i >= 1) {
                // the single P buffer is free once the previous P V has completed
                const bool okp = mbar_wait(&pvdone[(i - 1) & 1], ((i - 1) >> 1) & 1, abort, a.err);
                if (!__all_sync(0xFFFFFFFFu, okp)) {
                    live = false;
                    break;
                }
            }
            // P row of head h: two 16-byte core-matrix rows (keys 0-7 and 8-15)
            uint8_t *pb = p_s + (h >> 3) * 256 + (h & 7) * 16;
#pragma unroll
            for (int kc = 0; kc < NK / 8; ++kc)
                *reinterpret_cast<uint4 *>(pb + kc * 128) = make_uint4(
                    pack_bf16(p[8 * kc], p[8 * kc + 1]), pack_bf16(p[8 * kc + 2], p[8 * kc + 3]),
                    pack_bf16(p[8 * kc + 4], p[8 * kc + 5]),
                    pack_bf16(p[8 * kc + 6], p[8 * kc + 7]));
            fence_proxy_async();
            mbar_arrive(&pfull[bb]);
        }
        if (nonfinite) raise_error(a.err, LSA_DEVERR_NONFINITE);
        bool okf = live && mbar_wait(&pvdone[(n - 1) & 1], ((n - 1) >> 1) & 1, abort, a.err);
        if (__all_sync(0xFFFFFFFFu, okf)) {
            fence_after();
            const float inv = l > 0.f ? 1.f / l : 0.f;
            const float lse = l > 0.f ? (m_ref + log2f(l)) * 0.6931471805599453f : -INFINITY;
#pragma unroll 1
            for (int ch = 0; ch < DVH / 32; ++ch) {
                uint32_t ov[32];
                tmem_ld32(o_tmem + ch * 32, ov);
                tmem_wait_ld();
                if (a.n_split == 1) {
                    __nv_bfloat16 *o = a.out + (r * H + h) * (int64_t)512 + half * DVH + ch * 32;
#pragma unroll
                    for (int j = 0; j < 32; j += 8)
                        *reinterpret_cast<uint4 *>(o + j) = make_uint4(
                            pack_bf16(__uint_as_float(ov[j]) * inv, __uint_as_float(ov[j + 1]) * inv),
                            pack_bf16(__uint_as_float(ov[j + 2]) * inv, __uint_as_float(ov[j + 3]) * inv),
                            pack_bf16(__uint_as_float(ov[j + 4]) * inv, __uint_as_float(ov[j + 5]) * inv),
                            pack_bf16(__uint_as_float(ov[j + 6]) * inv, __uint_as_float(ov[j + 7]) * inv));
                } else {
                    float *o = a.part_o + ((r * H + h) * a.n_split + split) * (int64_t)512 +
                               half * DVH + ch * 32;
#pragma unroll
                    for (int j = 0; j < 32; j += 4)
                        *reinterpret_cast<float4 *>(o + j) = make_float4(
                            __uint_as_float(ov[j]) * inv, __uint_as_float(ov[j + 1]) * inv,
                            __uint_as_float(ov[j + 2]) * inv, __uint_as_float(ov[j + 3]) * inv);
                }
            }
            if (half == 0) {
                if (a.n_split == 1)
                    a.lse[r * H + h] = lse;
                else
                    a.part_lse[(r * H + h) * a.n_split + split] = lse;
            }
        }
    }

    // ---- tear-down: free TMEM once every role is done with it
    fence_before();
    __syncthreads();
    fence_after();
    if (warp == 5) {
        __syncwarp();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
    }
}

}  // namespace

int attend_tc_tile() { return NK; }

cudaError_t launch_attend_tc(const AttendArgs &a, int64_t rows, cudaStream_t s) {
    if (rows <= 0) return cudaSuccess;
    if (rows > 0x7FFFFFFF) return cudaErrorInvalidValue;
    const int64_t nb = rows / a.T;  // sequences
    if (nb * a.L_max >= 0x7FFFFFFFll) return cudaErrorInvalidValue;
    CUtensorMap cmap;
    if (!make_tmap_2d_bf16(&cmap, a.c, DQK, (uint64_t)(nb * a.L_max), 64, 1))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(hfa_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kSmemLaunch);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)rows, 2u, (unsigned)a.n_split);
    hfa_tc_kernel<<<grid, kThreads, kSmemLaunch, s>>>(cmap, a);
    return cudaGetLastError();
}

}  // namespace lsa
