// attend_bwd_tc.cu -- HFA backward on the tcgen05 tensor cores (64 heads per CTA).
//
// Paper: Sec. 2.2 (u_t = Attn over the latent rows c_s, s in S_t), Sec. 3.1 (S_t = sink U swa
// U S_sparse), Sec. 4.1.1 (HFA backward: gather for dQ, scatter-add of the row gradients),
// Table 2 (the training setting).  With z_s = scale q.c_s, p_s = exp(z_s - lse),
// dp_s = dout . c_s[0:512], D = dout . out and dz_s = scale p_s (dp_s - D):
//   dq   = sum_s dz_s c_s
//   dc_s += dz_s q + p_s dout   (the second term on the first 512 dims)
//
// One CTA per (query row, group of 64 heads) walks the row's virtual key list [sink | window |
// gathered] in tiles of 128 keys.  Every product is an M = 128 tcgen05 MMA with the tile's keys
// or 128 latent dims as M, bf16 operands, fp32 accumulators in tensor memory:
//   S^T  [keys x heads] = C Q_h^T           (A: key tile, K-major; B: Q_h, K-major; K = 576)
//   dP^T [keys x heads] = C[:, :512] dO_h^T (K = 512)
//   dQ^T [dims x heads] += C^T dZ^T         (A: the key tile read MN-major, 128 dims per MMA;
//                                            B: dZ^T in shared memory; K = 128 keys)
//   dC   [keys x 64 dims] = dZ^T Q_h + P^T dO_h  per 64-dim chunk (A: P^T / dZ^T in tensor
//                                            memory; B: Q_h / dO_h read MN-major; K = 64 heads)
// so the row gradients of a tile are complete over the CTA's 64 heads before they are added to
// the caller's buffer (two partial sums per key and query at 128 heads).
//
// Tensor memory (512 columns): [0, 64) S^T, then dC buffer A; [64, 128) dP^T, then dC buffer B;
// [128, 448) dQ^T, five 128-dim blocks x 64 heads, for the whole row; [448, 480) P^T and
// [480, 512) dZ^T as bf16 pairs.
// Shared memory: Q_h (9 chunks of 64 heads x 64 dims) and dO_h (8 chunks) for the whole row;
// a ring of two 32 KB slots, each a 128-key x 128-dim unit of the key tile (the fifth unit of a
// tile holds the last 64 dims); dZ^T (128 keys x 64 heads).  Every operand buffer is rows of
// 128 bytes in the 128-byte swizzle, so one layout serves the K-major and the MN-major reads.
// A tile's five units stream through the ring twice: for S / dP, then for dQ^T after the
// softmax has formed dZ.
//
// Warp roles:
//   warps 0-3, 8-11  two warpgroups over the tile's 128 key rows: P and dZ of 32 heads each
//               (bf16 into tensor memory, dZ^T also into shared memory), then the drain of the
//               tile's dC chunks, the even ones by the first group and the odd ones by the second
//               (tensor memory -> 16-byte vector reductions into the latent-row gradients, eight
//               lanes per 128 contiguous bytes of a row), and the dq store at the end;
//   warp 4      tensor-memory allocation; lane 0 issues every MMA.  In the second pass it issues
//               dQ^T of a unit as soon as the unit has landed and a dC chunk as soon as its
//               buffer is free, so neither the gathers nor the drain wait on the other;
//   warps 5-7   the tile positions (warp 5, one tile ahead) and the gathers (cp.async).
// Every wait is bounded; a role that gives up raises the abort flag, and the others leave.
#include <cuda.h>

#include "lsa_internal.cuh"
#include "tc_ptx.cuh"

namespace lsa {
namespace {

using namespace tc;

constexpr int DQK = 576;
constexpr int DV = 512;
constexpr int HG = 64;                   // heads per CTA (the N of S / dP / dQ^T)
constexpr int NKEY = 128;                // keys per tile (the M of S / dP / dC)
constexpr int kChunkQ = HG * 128;        // one 64-dim chunk of Q_h / dO_h: 8 KB
constexpr int kHalf = NKEY * 128;        // one 64-dim chunk of the key tile: 16 KB
constexpr int kSlot = 2 * kHalf;         // a 128-dim unit: 32 KB
constexpr int kRing = 2;
constexpr int kUnits = 5;                // units per pass (dims 0-127, ..., 512-575)
constexpr int kChunksDC = DQK / 64;      // 9 dC chunks per tile
constexpr int kPosBufs = 4;
// 12 warps: the register file is split over the SM's four sub-partitions, so 3 warps each
// leave 170 registers per thread (a 13th warp would cap every thread at 128)
constexpr int kThreads = 384;
constexpr int kMmaWarp = 4, kProdWarp0 = 5, kProdWarps = 3;
constexpr int kProdThreads = 32 * kProdWarps;  // 96
constexpr int kSoftThreads = 256;              // warps 0-3 and 8-11
constexpr int kBarProd = 1;
constexpr float kLog2e = 1.4426950408889634f;

// tensor-memory columns
constexpr uint32_t TS = 0, TDP = 64, TDQ = 128, TP = 448, TZ = 480;

// shared-memory layout (offsets from a 1024-byte aligned base)
constexpr int OFF_Q = 0;
constexpr int OFF_O = OFF_Q + 9 * kChunkQ;
constexpr int OFF_RING = OFF_O + 8 * kChunkQ;
constexpr int OFF_DZ = OFF_RING + kRing * kSlot;
constexpr int OFF_POS = OFF_DZ + NKEY * 128;
constexpr int OFF_LSE = OFF_POS + kPosBufs * NKEY * 4;
constexpr int OFF_D = OFF_LSE + HG * 4;
constexpr int OFF_BAR = OFF_D + HG * 4;
constexpr int kNumBars = 2 * kRing + 1 + 1 + 2 + 2 + kPosBufs + 1;
constexpr int OFF_MISC = OFF_BAR + kNumBars * 8;
constexpr int kSmemBytes = OFF_MISC + 16 + 1024;  // + alignment slack
static_assert(OFF_RING % 1024 == 0 && OFF_DZ % 1024 == 0 && OFF_O % 1024 == 0, "swizzle atoms");
static_assert(OFF_BAR % 8 == 0 && OFF_MISC % 8 == 0, "barriers");
static_assert(kSmemBytes <= 232448, "shared memory");

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

// Operand descriptors, 128-byte swizzle: K-major rows of 128 B with 8-row groups 1024 B apart;
// MN-major with 64-element atoms `lbo` bytes apart along M / N and 8-row K groups 1024 B apart.
__device__ __forceinline__ uint64_t kdesc(uint32_t addr) { return smem_desc(addr, 16, 1024, 2); }
__device__ __forceinline__ uint64_t mdesc(uint32_t addr, uint32_t lbo) {
    return smem_desc(addr, lbo, 1024, 2);
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
                 "r"(d)
                 : "memory");
}

// 16 lanes x 8 column groups of 8 (x8): thread t gets lanes t/4 and t/4 + 8, columns 8k + 2 (t % 4)
// and + 1 in registers 4k, 4k + 1 (first lane) and 4k + 2, 4k + 3 (second lane).
__device__ __forceinline__ void tmem_ld_16x256b_x8(uint32_t taddr, uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.16x256b.x8.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
          "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]),
          "=r"(v[13]), "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]),
          "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]),
          "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]),
          "=r"(v[31])
        : "r"(taddr));
}

// dst[0..3] += v, fire and forget (no value comes back, so nothing waits on the L2 round trip)
__device__ __forceinline__ void red_add_v4(float *dst, uint32_t a, uint32_t b, uint32_t c,
                                           uint32_t d) {
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(dst), "f"(__uint_as_float(a)),
                 "f"(__uint_as_float(b)), "f"(__uint_as_float(c)), "f"(__uint_as_float(d))
                 : "memory");
}

// Barrier over the producer warps that also ANDs a predicate across them.
__device__ __forceinline__ bool prod_and(bool p) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.and.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)p), "r"(kBarProd), "r"(kProdThreads)
        : "memory");
    return r != 0;
}

__global__ void __launch_bounds__(kThreads, 1) hfa_bwd_tc_kernel(BwdArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(sm);
    const uint32_t q_s = sbase + OFF_Q, o_s = sbase + OFF_O, ring_s = sbase + OFF_RING,
                   dz_s = sbase + OFF_DZ;
    int32_t *pos_s = reinterpret_cast<int32_t *>(sm + OFF_POS);  // [kPosBufs][NKEY]
    float *lse2_s = reinterpret_cast<float *>(sm + OFF_LSE);
    float *D_s = reinterpret_cast<float *>(sm + OFF_D);
    uint64_t *full = reinterpret_cast<uint64_t *>(sm + OFF_BAR);  // [kRing] unit landed
    uint64_t *empty = full + kRing;       // [kRing] the MMAs reading the unit completed
    uint64_t *sfull = empty + kRing;      // S^T and dP^T of the tile complete
    uint64_t *pready = sfull + 1;         // P^T / dZ^T written (128 arrivals)
    uint64_t *dcfull = pready + 1;        // [2] dC chunk complete in buffer A / B
    uint64_t *dcfree = dcfull + 2;        // [2] buffer A / B read out (128 arrivals)
    uint64_t *posready = dcfree + 2;      // [kPosBufs] tile positions written (32 arrivals)
    uint64_t *done = posready + kPosBufs; // every MMA of the row complete
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + OFF_MISC);
    volatile int *abort = reinterpret_cast<volatile int *>(sm + OFF_MISC + 4);
    int *nsp_s = reinterpret_cast<int *>(sm + OFF_MISC + 8);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t r = blockIdx.x;
    const int h0 = blockIdx.y * HG;
    const int64_t b = r / a.T;
    const int64_t t = a.q_pos[r];
    const int64_t len = a.kv_len[b];
    float *dq_row = a.dq + (r * a.H + h0) * (int64_t)DQK;
    if (!(t >= 0 && t < len && len <= a.L_max)) {
        if (tid == 0 && blockIdx.y == 0) raise_error(a.err, LSA_DEVERR_QPOS);
        // the row has no keys: its dq slice is written as zeros, no latent row is touched
        for (int i = tid; i < HG * DQK; i += kThreads) dq_row[i] = 0.f;
        return;
    }
    const Regions g = regions_of(t, a.Ks, a.Kw);
    const __nv_bfloat16 *cseq = a.c + b * a.L_max * DQK;

    if (warp == kMmaWarp) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32(tmem_slot)), "r"(512));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    if (tid == 0) {
        for (int i = 0; i < kRing; ++i) {
            mbar_init(&full[i], kProdThreads);
            mbar_init(&empty[i], 1);
        }
        mbar_init(sfull, 1);
        mbar_init(pready, kSoftThreads);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&dcfull[i], 1);
            mbar_init(&dcfree[i], 128);  // the warpgroup that drains the buffer
        }
        for (int i = 0; i < kPosBufs; ++i) mbar_init(&posready[i], 32);
        mbar_init(done, 1);
        *abort = 0;
        *nsp_s = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    {
        // the gathered picks of this row (ascending, -1 after the last)
        const int32_t *gidx = a.idx + r * a.K;
        int c = 0;
        for (int i = tid; i < a.K; i += kThreads) c += (gidx[i] >= 0);
        if (c) atomicAdd(nsp_s, c);
    }
    // Q_h and dO_h into their swizzled chunks: head n, dims 8u..8u+7 of chunk j at row n,
    // 16-byte unit u ^ (n & 7)
    {
        const uint4 *qg = reinterpret_cast<const uint4 *>(a.q + (r * a.H + h0) * (int64_t)DQK);
        for (int e = tid; e < HG * (DQK / 8); e += kThreads) {
            const int n = e / (DQK / 8), c8 = e - n * (DQK / 8), j = c8 >> 3, u = c8 & 7;
            const uint4 v = qg[e];
            st_shared_v4(q_s + j * kChunkQ + n * 128 + ((u ^ (n & 7)) << 4), v.x, v.y, v.z, v.w);
        }
        const uint4 *dg = reinterpret_cast<const uint4 *>(a.dout + (r * a.H + h0) * (int64_t)DV);
        for (int e = tid; e < HG * (DV / 8); e += kThreads) {
            const int n = e / (DV / 8), c8 = e - n * (DV / 8), j = c8 >> 3, u = c8 & 7;
            const uint4 v = dg[e];
            st_shared_v4(o_s + j * kChunkQ + n * 128 + ((u ^ (n & 7)) << 4), v.x, v.y, v.z, v.w);
        }
    }
    // the forward's lse (log2 units) and D = dout . out per head, one head per warp at a time
    for (int hh = warp; hh < HG; hh += kThreads / 32) {
        const uint4 *orow =
            reinterpret_cast<const uint4 *>(a.o + (r * a.H + h0 + hh) * (int64_t)DV) + lane * 2;
        const uint4 *drow =
            reinterpret_cast<const uint4 *>(a.dout + (r * a.H + h0 + hh) * (int64_t)DV) + lane * 2;
        float acc = 0.f;
#pragma unroll
        for (int v = 0; v < 2; ++v) {
            const uint4 ov = orow[v], dv = drow[v];
            const __nv_bfloat162 *o2 = reinterpret_cast<const __nv_bfloat162 *>(&ov);
            const __nv_bfloat162 *d2 = reinterpret_cast<const __nv_bfloat162 *>(&dv);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float2 of = __bfloat1622float2(o2[k]), df = __bfloat1622float2(d2[k]);
                acc = fmaf(of.x, df.x, fmaf(of.y, df.y, acc));
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, o);
        if (lane == 0) {
            const float ls = a.lse[r * a.H + h0 + hh];
            lse2_s[hh] = (ls > -INFINITY) ? ls * kLog2e : INFINITY;  // no keys: p = 0
            D_s[hh] = acc;
            if (!isfinite(acc) || ls != ls || ls == INFINITY) raise_error(a.err, LSA_DEVERR_NONFINITE);
        }
    }
    fence_proxy_async();  // the operand writes above, seen by the tensor cores
    fence_before();
    __syncthreads();
    fence_after();
    const uint32_t tmem = *tmem_slot;
    const int64_t n_sp = *nsp_s;
    const int64_t n_total = g.sink_hi + (g.swa_hi - g.swa_lo) + n_sp;
    const int n_tiles = (int)((n_total + NKEY - 1) / NKEY);
    const float sl2 = a.scale * kLog2e;

    if (warp < 4 || warp >= 8) {
        // ================================================= softmax, dC drain, dq store
        // Two warpgroups over the same 128 key rows (tensor-memory lane = row): group gr forms
        // P and dZ of heads 32 gr .. 32 gr + 31, then drains the dC chunks of its buffer (group
        // 0: buffer B, the even chunks; group 1: buffer A, the odd ones).
        const int gr = warp >> 3, quad = warp & 3;
        const int row = quad * 32 + lane;
        const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
        float *dc_seq = a.dc + b * a.L_max * DQK;
        const uint32_t tbuf = gr ? TS : TDP;        // the dC buffer this group drains
        uint64_t *bfull = &dcfull[gr ? 0 : 1], *bfree = &dcfree[gr ? 0 : 1];
        int uses = 0;
        bool live = true;
        for (int i = 0; i < n_tiles && live; ++i) {
            live = warp_wait(sfull, i & 1, abort, a.err) &&
                   warp_wait(&posready[i & (kPosBufs - 1)], (i / kPosBufs) & 1, abort, a.err);
            if (!live) break;
            fence_after();
            const int32_t *ptile = pos_s + (i & (kPosBufs - 1)) * NKEY;
            const bool valid = ptile[row] >= 0;
            {
                uint32_t sv[32], dv[32];
                tmem_ld32(tmem + lane_base + TS + gr * 32, sv);
                tmem_ld32(tmem + lane_base + TDP + gr * 32, dv);
                tmem_wait_ld();
                uint32_t pk[16], zk[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const int h = gr * 32 + 2 * e;
                    const float l0 = lse2_s[h], l1 = lse2_s[h + 1];
                    const float d0 = D_s[h], d1 = D_s[h + 1];
                    const float p0 = valid ? exp2f(fmaf(__uint_as_float(sv[2 * e]), sl2, -l0)) : 0.f;
                    const float p1 =
                        valid ? exp2f(fmaf(__uint_as_float(sv[2 * e + 1]), sl2, -l1)) : 0.f;
                    pk[e] = pack_bf16(p0, p1);
                    zk[e] = pack_bf16(p0 * (__uint_as_float(dv[2 * e]) - d0) * a.scale,
                                      p1 * (__uint_as_float(dv[2 * e + 1]) - d1) * a.scale);
                }
                tmem_st16(tmem + lane_base + TP + gr * 16, pk);
                tmem_st16(tmem + lane_base + TZ + gr * 16, zk);
                // dZ^T row in shared memory: this group's 32 heads are 16-byte units 4 gr .. +3
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const int u = gr * 4 + c;
                    st_shared_v4(dz_s + row * 128 + ((u ^ (row & 7)) << 4), zk[4 * c],
                                 zk[4 * c + 1], zk[4 * c + 2], zk[4 * c + 3]);
                }
            }
            tmem_wait_st();
            fence_proxy_async();
            fence_before();
            mbar_arrive(pready);
            // this group's dC chunks of the tile
            for (int j = gr; j < kChunksDC; j += 2) {
                if (!warp_wait(bfull, uses & 1, abort, a.err)) {
                    live = false;
                    break;
                }
                fence_after();
                // the chunk as two 16-row halves: thread t holds columns 8k + 2 (t % 4), +1 of
                // rows t/4 and t/4 + 8 of each half
                uint32_t w[2][32];
                tmem_ld_16x256b_x8(tmem + ((uint32_t)(quad * 32) << 16) + tbuf, w[0]);
                tmem_ld_16x256b_x8(tmem + ((uint32_t)(quad * 32 + 16) << 16) + tbuf, w[1]);
                tmem_wait_ld();
                fence_before();
                mbar_arrive(bfree);
                ++uses;
                // Three trades between lanes.  After the first (t, t ^ 1) the even lane holds,
                // for each column group k, four columns of the first row (8k + 4 (t % 4 / 2)
                // ..) and the odd lane the same columns of the second row; after the second
                // (t, t ^ 1) the even lane keeps the even groups of both rows and the odd lane
                // the odd ones, so four lanes hold 64 contiguous bytes of a row; after the third
                // (t, t ^ 4, between the lanes of neighbouring row pairs) eight lanes hold 128
                // contiguous bytes of one row per reduction instruction (a lane per row would
                // touch 32 rows).
                const bool odd = lane & 1, og = (lane >> 2) & 1;
                const int cq = 4 * ((lane & 3) >> 1);
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    const int ra = quad * 32 + hf * 16 + (lane >> 2), rb = ra + 8;
                    // rows of this lane's group and of its neighbour (ra ^ 1: the other group
                    // of the pair)
                    const int64_t pa = ptile[ra], pb = ptile[rb], pan = ptile[ra ^ 1],
                                  pbn = ptile[rb ^ 1];
                    uint32_t x[8][4];
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const uint32_t s0 = odd ? w[hf][4 * k] : w[hf][4 * k + 2];
                        const uint32_t s1 = odd ? w[hf][4 * k + 1] : w[hf][4 * k + 3];
                        const uint32_t r0 = __shfl_xor_sync(0xFFFFFFFFu, s0, 1);
                        const uint32_t r1 = __shfl_xor_sync(0xFFFFFFFFu, s1, 1);
                        x[k][0] = odd ? r0 : w[hf][4 * k];
                        x[k][1] = odd ? r1 : w[hf][4 * k + 1];
                        x[k][2] = odd ? w[hf][4 * k + 2] : r0;
                        x[k][3] = odd ? w[hf][4 * k + 3] : r1;
                    }
                    // after the second trade: va[m] / vb[m] = 16 bytes of the first / second row
                    // at columns 8 (2m + odd) + cq of the chunk
                    uint32_t va[4][4], vb[4][4];
#pragma unroll
                    for (int m = 0; m < 4; ++m) {
                        uint32_t y[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            y[e] = __shfl_xor_sync(0xFFFFFFFFu,
                                                   odd ? x[2 * m][e] : x[2 * m + 1][e], 1);
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            va[m][e] = odd ? y[e] : x[2 * m][e];
                            vb[m][e] = odd ? x[2 * m + 1][e] : y[e];
                        }
                    }
                    // third trade, per pair of m: the even group of a row pair keeps m = 2mp and
                    // takes the odd group's, the odd group keeps m = 2mp + 1 and takes the even
                    // group's
#pragma unroll
                    for (int mp = 0; mp < 2; ++mp) {
                        const int mo = og ? 2 * mp + 1 : 2 * mp;  // the m this lane writes
                        uint32_t ta[4], tb[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            ta[e] = __shfl_xor_sync(0xFFFFFFFFu,
                                                    og ? va[2 * mp][e] : va[2 * mp + 1][e], 4);
                            tb[e] = __shfl_xor_sync(0xFFFFFFFFu,
                                                    og ? vb[2 * mp][e] : vb[2 * mp + 1][e], 4);
                        }
                        // the even group's rows (1), then the odd group's (2)
                        uint32_t d1a[4], d2a[4], d1b[4], d2b[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const uint32_t oa = og ? va[2 * mp + 1][e] : va[2 * mp][e];
                            const uint32_t ob = og ? vb[2 * mp + 1][e] : vb[2 * mp][e];
                            d1a[e] = og ? ta[e] : oa;
                            d2a[e] = og ? oa : ta[e];
                            d1b[e] = og ? tb[e] : ob;
                            d2b[e] = og ? ob : tb[e];
                        }
                        const int col = j * 64 + 8 * (2 * mo + (odd ? 1 : 0)) + cq;
                        const int64_t r1a = og ? pan : pa, r2a = og ? pa : pan;
                        const int64_t r1b = og ? pbn : pb, r2b = og ? pb : pbn;
                        if (r1a >= 0) red_add_v4(dc_seq + r1a * DQK + col, d1a[0], d1a[1], d1a[2], d1a[3]);
                        if (r2a >= 0) red_add_v4(dc_seq + r2a * DQK + col, d2a[0], d2a[1], d2a[2], d2a[3]);
                        if (r1b >= 0) red_add_v4(dc_seq + r1b * DQK + col, d1b[0], d1b[1], d1b[2], d1b[3]);
                        if (r2b >= 0) red_add_v4(dc_seq + r2b * DQK + col, d2b[0], d2b[1], d2b[2], d2b[3]);
                    }
                }
            }
        }
        // dq: dQ^T block u holds dims 128 u + row (64 dims in the last block), heads by column;
        // group 0 stores blocks 0-2, group 1 blocks 3-4
        if (n_tiles == 0) {
            for (int i = gr * 128 + quad * 32 + lane; i < HG * DQK; i += kSoftThreads)
                dq_row[i] = 0.f;  // no keys
        } else if (live && warp_wait(done, 0, abort, a.err)) {
            fence_after();
#pragma unroll 1
            for (int u = gr ? 3 : 0; u < (gr ? kUnits : 3); ++u) {
                if (u == kUnits - 1 && quad >= 2) break;
                const int dim = u * 128 + row;
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    uint32_t v[32];
                    tmem_ld32(tmem + lane_base + TDQ + u * 64 + hf * 32, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int n = 0; n < 32; ++n)
                        dq_row[(int64_t)(hf * 32 + n) * DQK + dim] = __uint_as_float(v[n]);
                }
            }
        }
    } else if (warp == kMmaWarp) {
        // ================================================= MMA issuer
        if (lane == 0) {
            const uint32_t idesc_kk = (1u << 4) | (1u << 7) | (1u << 10) |
                                      ((uint32_t)(HG >> 3) << 17) | ((uint32_t)(NKEY >> 4) << 24);
            const uint32_t idesc_dq = idesc_kk | (1u << 15) | (1u << 16);
            const uint32_t idesc_dc = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) |
                                      ((uint32_t)(64 >> 3) << 17) | ((uint32_t)(NKEY >> 4) << 24);
            int q = 0, usesA = 0, usesB = 0;
            bool live = true;
            for (int i = 0; i < n_tiles && live; ++i) {
                if (i > 0) {
                    // S^T / dP^T overwrite dC buffers A / B: tile i - 1's last chunks read out
                    live = mbar_wait(&dcfree[0], (usesA - 1) & 1, abort, a.err) &&
                           mbar_wait(&dcfree[1], (usesB - 1) & 1, abort, a.err);
                    if (!live) break;
                    fence_after();
                }
                // ---- pass 1: S^T and dP^T over the five units
                for (int u = 0; u < kUnits; ++u) {
                    if (!(live = mbar_wait(&full[q & 1], (q >> 1) & 1, abort, a.err))) break;
                    fence_proxy_async();  // the cp.async writes of the unit, seen by the MMA
                    fence_after();
                    const uint32_t slot = ring_s + (q & 1) * kSlot;
                    for (int hf = 0; hf < (u < 4 ? 2 : 1); ++hf) {
                        const int j = 2 * u + hf;
                        const uint32_t ac = slot + hf * kHalf;
#pragma unroll
                        for (int k = 0; k < 4; ++k)
                            umma_bf16(tmem + TS, kdesc(ac + k * 32),
                                      kdesc(q_s + j * kChunkQ + k * 32), idesc_kk, (j | k) != 0);
                        if (j < 8) {
#pragma unroll
                            for (int k = 0; k < 4; ++k)
                                umma_bf16(tmem + TDP, kdesc(ac + k * 32),
                                          kdesc(o_s + j * kChunkQ + k * 32), idesc_kk,
                                          (j | k) != 0);
                        }
                    }
                    umma_commit(&empty[q & 1]);
                    ++q;
                }
                if (!live) break;
                umma_commit(sfull);
                if (!(live = mbar_wait(pready, i & 1, abort, a.err))) break;
                fence_after();
                // ---- pass 2: dQ^T of each unit as soon as it has landed (the gathers never wait
                // on the drain) and the dC chunks as soon as their buffer is free
                int u = 0, j = 0;
                uint64_t t_idle = 0;
                while (u < kUnits || j < kChunksDC) {
                    bool progressed = false;
                    if (u < kUnits && mbar_try(&full[q & 1], (q >> 1) & 1)) {
                        fence_proxy_async();
                        fence_after();
                        const uint32_t slot = ring_s + (q & 1) * kSlot;
#pragma unroll
                        for (int ks = 0; ks < NKEY / 16; ++ks)
                            umma_bf16(tmem + TDQ + u * 64, mdesc(slot + ks * 2048, kHalf),
                                      mdesc(dz_s + ks * 2048, kHalf), idesc_dq,
                                      (i > 0 || ks > 0));
                        umma_commit(&empty[q & 1]);
                        ++q;
                        ++u;
                        progressed = true;
                    }
                    if (j < kChunksDC) {
                        const bool inA = j & 1;
                        const int uses = inA ? usesA : usesB;
                        // the buffer's previous chunk of this tile has been read out (its last
                        // chunk of the tile before was waited for ahead of S^T / dP^T)
                        if (j < 2 || mbar_try(&dcfree[inA ? 0 : 1], (uses - 1) & 1)) {
                            fence_after();
                            const uint32_t d = tmem + (inA ? TS : TDP);
#pragma unroll
                            for (int ks = 0; ks < 4; ++ks)
                                umma_bf16_ts(d, tmem + TZ + ks * 8,
                                             mdesc(q_s + j * kChunkQ + ks * 2048, kChunkQ),
                                             idesc_dc, ks > 0);
                            if (j < 8) {
#pragma unroll
                                for (int ks = 0; ks < 4; ++ks)
                                    umma_bf16_ts(d, tmem + TP + ks * 8,
                                                 mdesc(o_s + j * kChunkQ + ks * 2048, kChunkQ),
                                                 idesc_dc, 1u);
                            }
                            umma_commit(&dcfull[inA ? 0 : 1]);
                            if (inA)
                                ++usesA;
                            else
                                ++usesB;
                            ++j;
                            progressed = true;
                        }
                    }
                    if (progressed) {
                        t_idle = 0;
                    } else if (t_idle == 0) {
                        t_idle = globaltimer();
                    } else if (*abort || globaltimer() - t_idle > kWaitNs) {
                        if (!*abort) raise_error(a.err, LSA_DEVERR_TIMEOUT);
                        live = false;
                        break;
                    }
                }
            }
            if (!live) *abort = 1;
            // every MMA issued has completed before the row's dq is read or the memory freed
            umma_commit(done);
            const uint64_t ts = globaltimer();
            while (!mbar_try(done, 0))
                if (globaltimer() - ts > kWaitNs) {
                    raise_error(a.err, LSA_DEVERR_TIMEOUT);
                    break;
                }
        }
    } else {
        // ================================================= positions and gathers
        const int pt = tid - 32 * kProdWarp0;  // 0 .. kProdThreads - 1
        const int32_t *idx = a.idx + r * a.K;
        auto positions = [&](int i) {  // warp kProdWarp0: the 128 positions of tile i
            int32_t *ps = pos_s + (i & (kPosBufs - 1)) * NKEY;
            for (int e = lane; e < NKEY; e += 32)
                ps[e] = (int32_t)bwd_key_pos(a.err, idx, g, n_sp, (int64_t)i * NKEY + e);
            mbar_arrive(&posready[i & (kPosBufs - 1)]);
        };
        if (warp == kProdWarp0 && n_tiles > 0) positions(0);
        int q = 0;
        bool ok = true;
        for (int i = 0; i < n_tiles; ++i) {
            if (!prod_and(ok && !*abort)) break;  // tile i's positions, seen by every producer
            const int32_t *ps = pos_s + (i & (kPosBufs - 1)) * NKEY;
            for (int pass = 0; pass < 2 && ok; ++pass) {
                for (int u = 0; u < kUnits; ++u) {
                    const int slot = q & 1;
                    if (q >= kRing && !(ok = warp_wait(&empty[slot], ((q >> 1) - 1) & 1, abort,
                                                       a.err)))
                        break;
                    // key row kr, 16-byte piece c of its 64-dim half hf: row kr of the half,
                    // unit c ^ (kr & 7); rows past the list are zero-filled
                    uint8_t *sb = sm + OFF_RING + slot * kSlot;
                    const int sh = (u < kUnits - 1) ? 4 : 3;  // log2 of the pieces per key
                    for (int e = pt; e < (NKEY << sh); e += kProdThreads) {
                        const int kr = e >> sh, pc = e & ((1 << sh) - 1), hf = pc >> 3, c = pc & 7;
                        const int64_t p = ps[kr];
                        cp_async16(sb + hf * kHalf + kr * 128 + ((c ^ (kr & 7)) << 4),
                                   cseq + (p >= 0 ? p : 0) * DQK + u * 128 + hf * 64 + c * 8,
                                   p >= 0 ? 16 : 0);
                    }
                    cp_async_arrive_noinc(&full[slot]);
                    ++q;
                }
                // the next tile's positions while this tile's second pass streams
                if (pass == 0 && warp == kProdWarp0 && i + 1 < n_tiles) positions(i + 1);
            }
        }
        cp_async_wait_all();  // nothing of this thread is in flight when the CTA leaves
    }
    fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
    }
}

}  // namespace

bool attend_bwd_tc_supported(const BwdArgs &a) {
    return a.H % HG == 0 && a.lse != nullptr && a.o != nullptr;
}

cudaError_t launch_attend_bwd_tc(const BwdArgs &a, int64_t rows, cudaStream_t s) {
    if (rows <= 0) return cudaSuccess;
    if (rows > 0x7FFFFFFF || !attend_bwd_tc_supported(a) || a.H / HG > 65535)
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(hfa_bwd_tc_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)rows, (unsigned)(a.H / HG));
    hfa_bwd_tc_kernel<<<grid, kThreads, kSmemBytes, s>>>(a);
    return launched();
}

}  // namespace lsa
