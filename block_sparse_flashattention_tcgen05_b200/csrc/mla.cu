// mla.cu -- split-KV MLA decode with softmax-threshold block skipping (BLASST)
// on tcgen05: one latent KV head of 576 columns (512 latent + 64 RoPE) shared
// by every query head; Q.K^T contracts all 576 columns, P.V uses the first
// 512 columns of the same cache rows as V.
//
// The tile is all G = Hq query heads x Lq queries (G*Lq <= 128 rows, one TMEM
// lane each); KV blocks of 64 keys.  The 128 x 512 fp32 output does not fit one
// SM's tensor memory next to S, so two CTAs share a (split, sequence): CTA h
// accumulates value columns 256h..256h+255.  Both compute the whole S = Q.K^T
// with the same sequence of tensor-core instructions on the same operands, so
// both hold bit-identical scores and take the same skip decisions without
// talking to each other; the second CTA's K reads are served by L2.  Per block
// the duplicated Q.K^T costs about as many tensor cycles as one block of K takes
// to stream from HBM, so the duplication does not lengthen the kernel while it
// removes any exchange of scores between SMs.
//
// Q (128 x 576 bf16) is split between tensor memory and shared memory: 64-column
// boxes 0..3 live in TMEM (A operand of tcgen05.mma from TMEM), boxes 4..8 in
// shared memory.  That leaves a 2-stage ring of whole K blocks (9 boxes, 72 KB).
//
// Warp roles (192 threads per CTA): warps 0-3 softmax/decision (thread = row),
// warp 4 TMA producer (Q boxes 4..8 once, each K block), warp 5 TMEM allocation
// + tcgen05.mma issue.
// TMEM: S [0,64), P [64,128) (two bf16 buffers: kept blocks alternate, so the
// softmax writes P(k) once the P.V of kept block k-2 is done), Q boxes 0..3
// [128,256) (bf16), O_half [256,512).
//
// Per block: S (always), tile decision as in the other kernels (true running
// max, restarted per split, first visited block kept); kept blocks: lazy O
// rescale, P = 2^(s - M_ref) -> bf16 in TMEM, O += P V_j.  Skipped blocks skip
// exp and P.V; their V bytes are K bytes already loaded (V adds no memory
// traffic in MLA).
#include <cuda_bf16.h>
#include <math_constants.h>

#include "internal.h"
#include "ptx.cuh"

namespace blasst {
namespace {

constexpr int kThreads = 192;
constexpr int kRows = 128;
constexpr int kBN = 64;
constexpr int kBoxes = 9;                       // 576 = 9 x 64 contraction columns
constexpr int kQTmemBoxes = 4;                  // Q boxes 0..3 in TMEM, 4..8 in shared memory
constexpr int kQBoxBytes = kRows * 128;         // 128 rows x 64 bf16
constexpr int kKBoxBytes = kBN * 128;           // 64 keys x 64 bf16
constexpr int kStages = 2;
constexpr int kKStageBytes = kBoxes * kKBoxBytes;                 // 72 KB
constexpr int kQSmemBytes = (kBoxes - kQTmemBoxes) * kQBoxBytes;  // 80 KB
constexpr uint32_t kColP = 64, kColQ = 128, kColO = 256;  // P buffer b at kColP + 32 b
constexpr float kRescaleThreshold = 8.0f;
constexpr int kStatusTimeout = 1;

struct MlaSmemTail {
    uint64_t k_full[kStages], k_empty[kStages];
    uint64_t q_full, qt_full, s_full, s_free, mma_done;
    uint64_t o_done[2];  // [P buffer]: the P.V that read it has completed
    // [block parity]: the softmax warps can publish block j+1 before the MMA warp
    // has taken block j, never further ahead
    uint64_t p_full[2];
    uint32_t tmem_base;
    int dec[2];
    int abort;
    float gred[4];
};

constexpr int mla_smem_bytes() {
    return kQSmemBytes + kStages * kKStageBytes + (int)sizeof(MlaSmemTail) + 1024;
}

__device__ __forceinline__ void set_timeout(MlaSmemTail *t, unsigned int *status) {
    t->abort = 1;
    if (status) atomicOr(status, kStatusTimeout);
}

template <bool CALIB>
__global__ void __launch_bounds__(kThreads, 1)
    mla_split_kernel(const MlaParams p, const __grid_constant__ CUtensorMap tmap_q,
                     const __grid_constant__ CUtensorMap tmap_k) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sq = smem;                 // Q boxes 4..8
    uint8_t *sk = smem + kQSmemBytes;   // K ring
    MlaSmemTail *tl = reinterpret_cast<MlaSmemTail *>(sk + kStages * kKStageBytes);

    const int half = blockIdx.x & 1;    // value columns 256*half .. +255
    const int split = blockIdx.x >> 1, b = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int j0 = split * p.per_split;
    const int j1 = min(p.nb, j0 + p.per_split);
    const int nblk = max(0, j1 - j0);
    // ring entries: [block 0 (seed)], then the split's blocks j0 .. j1-1
    const int seed = (p.seed && split > 0 && nblk > 0) ? 1 : 0;
    const int nent = nblk + seed;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kStages; i++) {
            mbar_init(&tl->k_full[i], 1);
            mbar_init(&tl->k_empty[i], 1);
        }
        mbar_init(&tl->q_full, 1);
        mbar_init(&tl->qt_full, 4);
        mbar_init(&tl->s_full, 1);
        mbar_init(&tl->s_free, 4);
        mbar_init(&tl->o_done[0], 1);
        mbar_init(&tl->o_done[1], 1);
        mbar_init(&tl->mma_done, 1);
        mbar_init(&tl->p_full[0], 4);
        mbar_init(&tl->p_full[1], 4);
        tl->abort = 0;
        fence_mbar_init();
    }
    if (warp == 5) {
        tmem_alloc(&tl->tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tl->tmem_base;

    if (warp == 4) {
        // ---------------------------------------------------------------- producer
        if (lane == 0 && nblk > 0) {
            tma_prefetch_desc(&tmap_q);
            tma_prefetch_desc(&tmap_k);
            mbar_arrive_expect_tx(&tl->q_full, kQSmemBytes);
            for (int x = kQTmemBoxes; x < kBoxes; x++)
                tma_load_3d(sq + (x - kQTmemBoxes) * kQBoxBytes, &tmap_q, &tl->q_full, x * 64, 0, b);
            int issued = 0;
            for (int e = 0; e < nent && !tl->abort; e++) {
                const int st = e % kStages;
                if (e >= kStages && !mbar_wait(&tl->k_empty[st], ((e / kStages) & 1) ^ 1, &tl->abort)) {
                    set_timeout(tl, p.status);
                    break;
                }
                const int blk = (seed && e == 0) ? 0 : j0 + e - seed;
                mbar_arrive_expect_tx(&tl->k_full[st], kKStageBytes);
                for (int x = 0; x < kBoxes; x++)
                    tma_load_3d(sk + st * kKStageBytes + x * kKBoxBytes, &tmap_k, &tl->k_full[st], x * 64,
                                blk * kBN, b);
                issued++;
            }
            mbar_wait(&tl->q_full, 0, nullptr);  // Q landed before this warp moves on
            if (tl->abort) {  // let copies already issued land
                for (int jj = max(0, issued - kStages); jj < issued; jj++)
                    mbar_wait(&tl->k_full[jj % kStages], (jj / kStages) & 1, nullptr);
            }
        }
    } else if (warp == 5) {
        // ------------------------------------------------------------- MMA issuer
        if (lane == 0 && nblk > 0) {
            constexpr uint32_t idesc_s = umma_idesc_bf16(128, kBN, 0);
            constexpr uint32_t idesc_pv = umma_idesc_bf16(128, 256, 1);
            constexpr uint32_t dhi = umma_desc_hi_sw128();
            const uint32_t q_lo = umma_desc_lo(smem_addr(sq), 16);
            const uint32_t k_lo = umma_desc_lo(smem_addr(sk), 16);
            // V = value columns 256*half.. = K boxes 4*half .. 4*half+3 of the stage, MN-major
            const uint32_t v_lo = umma_desc_lo(smem_addr(sk + half * 4 * kKBoxBytes), kKBoxBytes);
            const uint32_t s_col = tmem, p_col = tmem + kColP, q_col = tmem + kColQ, o_col = tmem + kColO;
            bool ok = mbar_wait(&tl->q_full, 0, &tl->abort) && mbar_wait(&tl->qt_full, 0, &tl->abort);
            if (!ok) set_timeout(tl, p.status);
            auto issue_s = [&](int jj) {  // S = Q . K_jj^T over all 576 columns, box 0 starts the sum
                const uint32_t kst = k_lo + (uint32_t)(((jj % kStages) * kKStageBytes) >> 4);
#pragma unroll
                for (int x = 0; x < kQTmemBoxes; x++)
#pragma unroll
                    for (int kk = 0; kk < 4; kk++)
                        umma_ts2(s_col, q_col + (uint32_t)(x * 32 + kk * 8),
                                 kst + (uint32_t)((x * kKBoxBytes + kk * 32) >> 4), dhi, idesc_s, (x | kk) ? 1u : 0u);
#pragma unroll
                for (int x = kQTmemBoxes; x < kBoxes; x++)
#pragma unroll
                    for (int kk = 0; kk < 4; kk++)
                        umma_ss2(s_col, q_lo + (uint32_t)(((x - kQTmemBoxes) * kQBoxBytes + kk * 32) >> 4),
                                 kst + (uint32_t)((x * kKBoxBytes + kk * 32) >> 4), dhi, idesc_s, 1u);
                umma_commit(&tl->s_full);
            };
            // Two independent streams over the ring entries, taken in whichever order they
            // become ready: S(ns) once the softmax holds S(ns-1) in registers and K(ns) has
            // landed, and entry np's decision (P.V when kept, then the K stage back to the
            // producer).  S(ns) never waits for a decision: holding it back until the P.V
            // of block ns-1 is issued (so that the stage is released sooner) leaves the
            // tensor pipe idle while the softmax works, and measured slower (1.31 against
            // 1.16 ms dense).  (S goes out as one uninterrupted run of 36 instructions:
            // pausing the issue between its boxes stalls the accumulation chain and costs
            // more than it saves.)
            int n_pv = 0, ns = 0, np = 0;
            long long t_last = clock64();
            while (ok && np < nent) {
                bool did = false;
                if (ns < nent && (ns == 0 || mbar_test_wait(&tl->s_free, (ns - 1) & 1)) &&
                    mbar_test_wait(&tl->k_full[ns % kStages], (ns / kStages) & 1)) {
                    tc_fence_after();
                    issue_s(ns);
                    ns++;
                    did = true;
                }
                if (np < ns && mbar_test_wait(&tl->p_full[np & 1], (np >> 1) & 1)) {
                    tc_fence_after();
                    if (!CALIB && tl->dec[np & 1]) {
                        const uint32_t vst = v_lo + (uint32_t)(((np % kStages) * kKStageBytes) >> 4);
#pragma unroll
                        for (int kk = 0; kk < kBN / 16; kk++)
                            umma_ts2(o_col, p_col + (uint32_t)((n_pv & 1) * 32 + kk * 8),
                                     vst + (uint32_t)((kk * 16 * 128) >> 4), dhi, idesc_pv,
                                     (n_pv > 0 || kk > 0) ? 1u : 0u);
                        umma_commit(&tl->o_done[n_pv & 1]);
                        n_pv++;
                    }
                    umma_commit(&tl->k_empty[np % kStages]);
                    np++;
                    did = true;
                }
                if (did) {
                    t_last = clock64();
                } else if (tl->abort || clock64() - t_last > kWaitLimitCycles) {
                    set_timeout(tl, p.status);
                    ok = false;
                }
            }
            umma_commit(&tl->mma_done);
            if (!mbar_wait(&tl->mma_done, 0, nullptr)) set_timeout(tl, p.status);
        }
        __syncwarp();
    } else if (nblk > 0) {
        // ----------------------------------------------------- softmax / decision
        const int row = threadIdx.x;  // 0..127, TMEM lane
        const bool valid_row = row < p.R;
        const int pos = row % p.Lq;
        const int last_key = !valid_row ? -1 : (p.causal ? pos + p.Lk - p.Lq : p.Lk - 1);
        const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
        const uint32_t s_addr = tmem + lane_off, o_addr = tmem + lane_off + kColO;
        // Q boxes 0..3 of this row -> TMEM, packed bf16 pairs
        {
            const uint16_t *qrow = p.q + ((size_t)b * p.R + (valid_row ? row : 0)) * 576;
#pragma unroll 1
            for (int x = 0; x < kQTmemBoxes; x++) {
                uint32_t w[32];
                const uint4 *src = reinterpret_cast<const uint4 *>(qrow + x * 64);
#pragma unroll
                for (int i = 0; i < 8; i++) {
                    const uint4 v = valid_row ? __ldg(src + i) : make_uint4(0u, 0u, 0u, 0u);
                    w[4 * i] = v.x;
                    w[4 * i + 1] = v.y;
                    w[4 * i + 2] = v.z;
                    w[4 * i + 3] = v.w;
                }
                tmem_st32(tmem + lane_off + kColQ + (uint32_t)(x * 32), w);
            }
            tc_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tl->qt_full);
        }
        const float NEG_INF = -CUDART_INF_F;
        const bool report = half == 0;  // one CTA of the pair writes mask, count and gaps
        float m_true = NEG_INF, m_ref = NEG_INF, l = 0.f, lr = 0.f;
        int n_kept = 0;
        unsigned int n_skip = 0;
        uint32_t mword = 0;
        int mword_idx = -1;
        for (int e = 0; e < nent; e++) {
            const int jj = e - seed;          // block index within the split; -1: the seed block
            const int j = jj < 0 ? 0 : j0 + jj;
            const int sl = e & 1;
            if (!mbar_wait(&tl->s_full, e & 1, &tl->abort)) set_timeout(tl, p.status);
            tc_fence_after();
            float s[64];
            {
                uint32_t *sr = reinterpret_cast<uint32_t *>(s);
                tmem_ld32(s_addr, sr);
                tmem_ld32(s_addr + 32, sr + 32);
                tc_wait_ld();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tl->s_free);  // S(jj+1) may overwrite it now

            const int lim = last_key - j * kBN;
            if (lim < kBN - 1) {
#pragma unroll
                for (int c = 0; c < kBN; c++)
                    if (c > lim) s[c] = NEG_INF;
            }
            float m0 = NEG_INF, m1 = NEG_INF, m2 = NEG_INF, m3 = NEG_INF;
#pragma unroll
            for (int c = 0; c < kBN; c += 8) {
                m0 = fmax3(m0, s[c], s[c + 1]);
                m1 = fmax3(m1, s[c + 2], s[c + 3]);
                m2 = fmax3(m2, s[c + 4], s[c + 5]);
                m3 = fmax3(m3, s[c + 6], s[c + 7]);
            }
            const float mt = fmax3(m0, m1, fmaxf(m2, m3)) * p.scale_log2;
            if (jj < 0) {
                // the seed block: its row maxima start the running max of this split; no
                // decision, no exp, no P.V, nothing reported
                m_true = mt;
                if (row == 0) tl->dec[sl] = 0;
                __syncwarp();
                if (lane == 0) mbar_arrive(&tl->p_full[sl]);
                continue;
            }
            const float mn = fmaxf(m_true, mt);
            const bool vote = (mt == NEG_INF) || (mt - mn < p.thr_log2);
            // (every block below Lk is visited: the last query row sees all keys)
            const bool all = bar_and(1, 128, vote);
            const bool first = jj == 0 && !seed;  // a seeded split has no forced first block
            const bool skip = all && !first;
            const bool kept = !skip;
            if (CALIB && report && p.gaps) {
                float g = mt == NEG_INF ? NEG_INF : mt - mn;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) g = fmaxf(g, __shfl_xor_sync(0xffffffffu, g, o));
                if (lane == 0) tl->gred[warp] = g;
                bar_sync(1, 128);
                if (row == 0) {
                    const float gg = fmaxf(fmaxf(tl->gred[0], tl->gred[1]), fmaxf(tl->gred[2], tl->gred[3]));
                    p.gaps[(size_t)b * p.nb + j] = first ? CUDART_INF_F : gg * 0.69314718055994531f;
                }
                bar_sync(1, 128);
            }
            if (row == 0) tl->dec[sl] = kept ? 1 : 0;
            if (!kept || CALIB) {
                if (kept) m_true = mn;
                __syncwarp();
                if (lane == 0) mbar_arrive(&tl->p_full[sl]);
            } else {
                m_true = mn;
                const bool warp_need = __any_sync(0xffffffffu, mn - m_ref > kRescaleThreshold);
                float alpha = 1.f;
                if (warp_need) {
                    alpha = (m_ref == NEG_INF || mn == NEG_INF) ? (mn == NEG_INF ? 1.f : 0.f) : ex2(m_ref - mn);
                    l *= alpha;
                    lr *= alpha;
                    if (mn != NEG_INF) m_ref = mn;
                }
                const float mref = m_ref == NEG_INF ? 0.f : m_ref;
                // Kept blocks alternate between two P buffers: buffer n_kept & 1 was last read by
                // the P.V of kept block n_kept - 2.  Rescaling O needs every earlier P.V done
                // (they complete in issue order).
                const int pbuf = n_kept & 1;
                if (warp_need && n_kept > 0) {
                    if (!mbar_wait(&tl->o_done[(n_kept - 1) & 1], ((n_kept - 1) >> 1) & 1, &tl->abort))
                        set_timeout(tl, p.status);
                    tc_fence_after();
                } else if (n_kept >= 2) {
                    if (!mbar_wait(&tl->o_done[pbuf], ((n_kept - 2) >> 1) & 1, &tl->abort)) set_timeout(tl, p.status);
                    tc_fence_after();
                }
                const uint32_t p_addr = tmem + lane_off + kColP + (uint32_t)(pbuf * 32);
                float rs = 0.f, rr = 0.f;
#pragma unroll
                for (int h = 0; h < 2; h++) {
                    uint32_t pk[16];
#pragma unroll
                    for (int c = 0; c < 16; c++) {
                        const float p0 = ex2(fmaf(s[h * 32 + 2 * c], p.scale_log2, -mref));
                        const float p1 = ex2(fmaf(s[h * 32 + 2 * c + 1], p.scale_log2, -mref));
                        pk[c] = pack_bf16x2(p0, p1);
                        rs += p0 + p1;
                        rr += __uint_as_float(pk[c] << 16) + __uint_as_float(pk[c] & 0xFFFF0000u);
                    }
                    tmem_st16(p_addr + h * 16, pk);
                }
                l += rs;
                lr += rr;
                if (warp_need && n_kept > 0) {
#pragma unroll 1
                    for (int c = 0; c < 8; c++) {
                        uint32_t orr[32];
                        tmem_ld32(o_addr + c * 32, orr);
                        tc_wait_ld();
#pragma unroll
                        for (int i = 0; i < 32; i++) orr[i] = __float_as_uint(__uint_as_float(orr[i]) * alpha);
                        tmem_st32(o_addr + c * 32, orr);
                    }
                }
                tc_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&tl->p_full[sl]);
                n_kept++;
            }
            if (skip) n_skip++;
            if (row == 0 && report && p.skip_mask && skip) {
                if (mword_idx != (j >> 5)) {
                    if (mword_idx >= 0 && mword) atomicOr(p.skip_mask + (size_t)b * p.words + mword_idx, mword);
                    mword_idx = j >> 5;
                    mword = 0;
                }
                mword |= 1u << (j & 31);
            }
        }
        if (row == 0 && report) {
            if (p.skip_mask && mword_idx >= 0 && mword) atomicOr(p.skip_mask + (size_t)b * p.words + mword_idx, mword);
            if (p.split_skips)
                p.split_skips[(size_t)b * p.num_splits + split] = n_skip;
            else if (p.skip_count && n_skip)
                atomicAdd(p.skip_count, (unsigned long long)n_skip);
        }
        if (!CALIB) {
            // split epilogue: normalised partial O (this CTA's 256 value columns), the split's lse
            const size_t orow = ((size_t)b * p.R + row) * p.num_splits + split;
            if (n_kept > 0) {
                if (!mbar_wait(&tl->o_done[(n_kept - 1) & 1], ((n_kept - 1) >> 1) & 1, &tl->abort))
                    set_timeout(tl, p.status);
                tc_fence_after();
            }
            const float inv = lr > 0.f ? 1.f / lr : 0.f;
#pragma unroll 1
            for (int c = 0; c < 8; c++) {
                uint32_t orr[32];
                tmem_ld32(o_addr + c * 32, orr);
                tc_wait_ld();
                if (valid_row) {
                    float *dst = p.part_o + orow * 512 + half * 256 + c * 32;
#pragma unroll
                    for (int i = 0; i < 32; i += 4) {
                        float4 v4;
                        v4.x = n_kept ? __uint_as_float(orr[i]) * inv : 0.f;
                        v4.y = n_kept ? __uint_as_float(orr[i + 1]) * inv : 0.f;
                        v4.z = n_kept ? __uint_as_float(orr[i + 2]) * inv : 0.f;
                        v4.w = n_kept ? __uint_as_float(orr[i + 3]) * inv : 0.f;
                        *reinterpret_cast<float4 *>(dst + i) = v4;
                    }
                }
            }
            if (valid_row && half == 0)
                p.part_lse[orow] = l > 0.f ? (m_ref + __log2f(l)) * 0.69314718055994531f : NEG_INF;
        }
    } else if (!CALIB) {
        // an empty split: its partial output is empty (lse = -inf) and the combine ignores it
        const int row = threadIdx.x;
        if (row < p.R) {
            const size_t orow = ((size_t)b * p.R + row) * p.num_splits + split;
            float *dst = p.part_o + orow * 512 + half * 256;
            for (int i = 0; i < 256; i += 4) *reinterpret_cast<float4 *>(dst + i) = make_float4(0.f, 0.f, 0.f, 0.f);
            if (half == 0) p.part_lse[orow] = -CUDART_INF_F;
        }
        if (half == 0 && threadIdx.x == 0 && p.split_skips) p.split_skips[(size_t)b * p.num_splits + split] = 0;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 5) tmem_dealloc(tmem, 512);
}

template <bool CALIB>
cudaError_t launch_t(const MlaParams &p, const CUtensorMap &tq, const CUtensorMap &tk, cudaStream_t st) {
    constexpr int smem = mla_smem_bytes();
    auto kern = mla_split_kernel<CALIB>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    dim3 grid(2 * p.num_splits, 1, p.B);
    kern<<<grid, kThreads, smem, st>>>(p, tq, tk);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_mla(const MlaParams &p, const CUtensorMap &tq, const CUtensorMap &tk, bool calib,
                       cudaStream_t st) {
    return calib ? launch_t<true>(p, tq, tk, st) : launch_t<false>(p, tq, tk, st);
}

}  // namespace blasst
