// mla.cu -- split-KV MLA decode with softmax-threshold block skipping (BLASST)
// on tcgen05: one latent KV head of 576 columns (512 latent + 64 RoPE) shared
// by every query head; Q.K^T contracts all 576 columns, P.V uses the first
// 512 columns of the same cache rows as V.
//
// The tile is all G = Hq query heads x Lq queries (G*Lq <= 128 rows, one TMEM
// lane each); KV blocks of 64 keys.  Per block: S (always), the tile decision
// as in the other kernels (true running max, restarted per split, first visited
// block kept); kept blocks: lazy O rescale, P = 2^(s - M_ref) -> bf16, O += P V_j.
// Skipped blocks skip exp and P.V; their V bytes are K bytes already loaded (V
// adds no memory traffic in MLA).
//
// Two kernels:
//   mla_calib_kernel  the decision-only pass (gaps, mask, count): one CTA per
//                     (split, sequence), S for every block, no V, no P;
//   mla_pair_kernel   the attention pass: a cluster of two CTAs per (split,
//                     sequence) that take turns computing S and exchange row
//                     maxima and P through distributed shared memory (below).
// Both compute S with the same sequence of tensor-core instructions -- Q boxes
// 0..5 from tensor memory, 6..8 from shared memory, contraction in box order --
// so the two passes see bit-identical scores and take identical decisions.
#include <cuda_bf16.h>
#include <math_constants.h>

#include "internal.h"
#include "ptx.cuh"

namespace blasst {
namespace {

constexpr int kRows = 128;
constexpr int kBN = 64;
constexpr int kBoxes = 9;                       // 576 = 9 x 64 contraction columns
constexpr int kQTmem = 6;                       // Q boxes 0..5 in TMEM, 6..8 in shared memory
constexpr int kQBoxBytes = kRows * 128;         // 128 rows x 64 bf16
constexpr int kKBoxBytes = kBN * 128;           // 64 keys x 64 bf16
constexpr int kQSmemBytes = (kBoxes - kQTmem) * kQBoxBytes;  // 48 KB
constexpr float kRescaleThreshold = 8.0f;
constexpr int kStatusTimeout = 1;

// ===================================================================== calibration
namespace calib {

constexpr int kThreads = 192;                   // warps 0-3 decision, 4 TMA, 5 TMEM + MMA
constexpr int kStages = 2;
constexpr int kKStageBytes = kBoxes * kKBoxBytes;  // 72 KB
constexpr uint32_t kColS = 0, kColQ = 64;

struct Tail {
    uint64_t k_full[kStages], k_empty[kStages];
    uint64_t q_full, qt_full, s_full, s_free, mma_done;
    uint32_t tmem_base;
    int abort;
    float gred[4];
};

constexpr int smem_bytes() { return kQSmemBytes + kStages * kKStageBytes + (int)sizeof(Tail) + 1024; }

__device__ __forceinline__ void set_timeout(Tail *t, unsigned int *status) {
    t->abort = 1;
    if (status) atomicOr(status, kStatusTimeout);
}

__global__ void __launch_bounds__(kThreads, 1)
    mla_calib_kernel(const MlaParams p, const __grid_constant__ CUtensorMap tmap_q,
                     const __grid_constant__ CUtensorMap tmap_k) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sq = smem;                 // Q boxes 6..8
    uint8_t *sk = smem + kQSmemBytes;   // K ring
    Tail *tl = reinterpret_cast<Tail *>(sk + kStages * kKStageBytes);

    const int split = blockIdx.x, b = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int j0 = split * p.per_split;
    const int j1 = min(p.nb, j0 + p.per_split);
    const int nblk = max(0, j1 - j0);

    if (threadIdx.x == 0) {
        for (int i = 0; i < kStages; i++) {
            mbar_init(&tl->k_full[i], 1);
            mbar_init(&tl->k_empty[i], 1);
        }
        mbar_init(&tl->q_full, 1);
        mbar_init(&tl->qt_full, 4);
        mbar_init(&tl->s_full, 1);
        mbar_init(&tl->s_free, 4);
        mbar_init(&tl->mma_done, 1);
        tl->abort = 0;
        fence_mbar_init();
    }
    if (warp == 5) {
        tmem_alloc(&tl->tmem_base, 256);
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
            for (int x = kQTmem; x < kBoxes; x++)
                tma_load_3d(sq + (x - kQTmem) * kQBoxBytes, &tmap_q, &tl->q_full, x * 64, 0, b);
            int issued = 0;
            for (int jj = 0; jj < nblk && !tl->abort; jj++) {
                const int st = jj % kStages;
                if (jj >= kStages && !mbar_wait(&tl->k_empty[st], ((jj / kStages) & 1) ^ 1, &tl->abort)) {
                    set_timeout(tl, p.status);
                    break;
                }
                mbar_arrive_expect_tx(&tl->k_full[st], kKStageBytes);
                for (int x = 0; x < kBoxes; x++)
                    tma_load_3d(sk + st * kKStageBytes + x * kKBoxBytes, &tmap_k, &tl->k_full[st], x * 64,
                                (j0 + jj) * kBN, b);
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
            constexpr uint32_t dhi = umma_desc_hi_sw128();
            const uint32_t q_lo = umma_desc_lo(smem_addr(sq), 16);
            const uint32_t k_lo = umma_desc_lo(smem_addr(sk), 16);
            const uint32_t s_col = tmem + kColS, q_col = tmem + kColQ;
            bool ok = mbar_wait(&tl->q_full, 0, &tl->abort) && mbar_wait(&tl->qt_full, 0, &tl->abort);
            if (!ok) set_timeout(tl, p.status);
            for (int jj = 0; jj < nblk && ok; jj++) {
                const int st = jj % kStages;
                if (!mbar_wait(&tl->k_full[st], (jj / kStages) & 1, &tl->abort) ||
                    (jj > 0 && !mbar_wait(&tl->s_free, (jj - 1) & 1, &tl->abort))) {
                    set_timeout(tl, p.status);
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t kst = k_lo + (uint32_t)((st * kKStageBytes) >> 4);
#pragma unroll
                for (int x = 0; x < kBoxes; x++)
#pragma unroll
                    for (int kk = 0; kk < 4; kk++) {
                        const uint32_t kd = kst + (uint32_t)((x * kKBoxBytes + kk * 32) >> 4);
                        if (x < kQTmem)
                            umma_ts2(s_col, q_col + (uint32_t)(x * 32 + kk * 8), kd, dhi, idesc_s, (x | kk) ? 1u : 0u);
                        else
                            umma_ss2(s_col, q_lo + (uint32_t)(((x - kQTmem) * kQBoxBytes + kk * 32) >> 4), kd, dhi,
                                     idesc_s, 1u);
                    }
                umma_commit(&tl->s_full);
                umma_commit(&tl->k_empty[st]);
            }
            umma_commit(&tl->mma_done);
            if (!mbar_wait(&tl->mma_done, 0, nullptr)) set_timeout(tl, p.status);
        }
        __syncwarp();
    } else if (nblk > 0) {
        // ------------------------------------------------------------ decisions
        const int row = threadIdx.x;  // 0..127, TMEM lane
        const bool valid_row = row < p.R;
        const int pos = row % p.Lq;
        const int last_key = !valid_row ? -1 : (p.causal ? pos + p.Lk - p.Lq : p.Lk - 1);
        const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
        {  // Q boxes 0..5 of this row -> TMEM, packed bf16 pairs
            const uint16_t *qrow = p.q + ((size_t)b * p.R + (valid_row ? row : 0)) * 576;
#pragma unroll 1
            for (int x = 0; x < kQTmem; x++) {
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
        float m_true = NEG_INF;
        unsigned int n_skip = 0;
        uint32_t mword = 0;
        int mword_idx = -1;
        for (int jj = 0; jj < nblk; jj++) {
            const int j = j0 + jj;
            if (!mbar_wait(&tl->s_full, jj & 1, &tl->abort)) set_timeout(tl, p.status);
            tc_fence_after();
            float s[64];
            {
                uint32_t *sr = reinterpret_cast<uint32_t *>(s);
                tmem_ld32(tmem + lane_off + kColS, sr);
                tmem_ld32(tmem + lane_off + kColS + 32, sr + 32);
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
            const float mn = fmaxf(m_true, mt);
            const bool vote = (mt == NEG_INF) || (mt - mn < p.thr_log2);
            // (every block below Lk is visited: the last query row sees all keys)
            const bool all = bar_and(1, 128, vote);
            const bool first = jj == 0;
            const bool skip = all && !first;
            if (p.gaps) {
                float g = mt == NEG_INF ? NEG_INF : mt - mn;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) g = fmaxf(g, __shfl_xor_sync(0xffffffffu, g, o));
                if (lane == 0) tl->gred[warp] = g;
                bar_sync(2, 128);
                if (row == 0) {
                    const float gg = fmaxf(fmaxf(tl->gred[0], tl->gred[1]), fmaxf(tl->gred[2], tl->gred[3]));
                    p.gaps[(size_t)b * p.nb + j] = first ? CUDART_INF_F : gg * 0.69314718055994531f;
                }
                bar_sync(2, 128);
            }
            if (!skip) m_true = mn;
            if (skip) {
                n_skip++;
                if (row == 0 && p.skip_mask) {
                    if (mword_idx != (j >> 5)) {
                        if (mword_idx >= 0 && mword) atomicOr(p.skip_mask + (size_t)b * p.words + mword_idx, mword);
                        mword_idx = j >> 5;
                        mword = 0;
                    }
                    mword |= 1u << (j & 31);
                }
            }
        }
        if (row == 0) {
            if (p.skip_mask && mword_idx >= 0 && mword) atomicOr(p.skip_mask + (size_t)b * p.words + mword_idx, mword);
            if (p.skip_count && n_skip) atomicAdd(p.skip_count, (unsigned long long)n_skip);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 5) tmem_dealloc(tmem, 256);
}

}  // namespace calib

// ===================================================================== pair kernel
// The attention pass.  A cluster of two CTAs (ranks h = 0, 1) shares a (split,
// sequence); CTA h accumulates value columns 256h .. 256h + 255 of O in its tensor
// memory.  Instead of both CTAs computing every S = Q.K^T, the two take the blocks
// of the split in turn: CTA h computes S, the block row maxima and P for the blocks
// jj (index within the split) with jj % 2 == h, and hands the other CTA what it
// needs through distributed shared memory:
//   - the block's row maxima (128 floats), so that both CTAs hold every block's
//     maxima, hence the same running max, the same skip decisions and the same
//     lazy exp reference (all of them functions of the maxima alone);
//   - for a kept block, P itself (128 x 64 bf16, 16 KB), by one bulk copy from the
//     owner's shared memory into the other CTA's, where it is the A operand of
//     that CTA's P.V.
// Each CTA keeps the row sums of its own blocks' P; the two partial sums are added
// at the end.  The tensor work per block drops from two S products (one per CTA)
// to one, and a CTA loads the whole block (all 9 boxes) only for its own blocks;
// for the other CTA's blocks it loads just its 4 value boxes (the owner's load of
// the same bytes has brought them into L2).
//
// Shared memory (one CTA per SM): Q boxes 6..8 (48 KB; boxes 0..5 live in tensor
// memory), one stage of the 5 boxes only S reads (40 KB), a 3-stage ring of this
// CTA's 4 value boxes of every block (96 KB), the own P staging tile (16 KB) and
// the partner's P tile (16 KB).
// TMEM: S [0,64), Q boxes 0..5 [64,256) (bf16 pairs), O half [256,512).
// Warps: 0-3 softmax/decision (thread = row), 4 TMA producer, 5 TMEM + MMA issue.
namespace pair {

constexpr int kThreads = 192;
constexpr int kSPartBytes = 5 * kKBoxBytes;            // the other half's 4 latent boxes + the RoPE box
constexpr int kVHalfBytes = 4 * kKBoxBytes;            // this CTA's 4 value boxes
constexpr int kNV = 3;                                 // value-box ring stages
constexpr int kPBytes = kRows * kBN * 2;               // 128 rows x 64 keys bf16
constexpr int kMx = 4;                                 // row-max exchange slots
constexpr int kDec = 4;                                // decisions in flight to the MMA thread
constexpr uint32_t kColS = 0, kColQ = 64, kColO = 256;

struct Tail {
    uint64_t q_full, qt_full, sp_full, sp_empty;
    uint64_t v_full[kNV], v_empty[kNV];
    uint64_t s_full, s_free, o_done, own_pv_done, mma_done;
    uint64_t p_ready[kDec], dec_free[kDec];
    uint64_t pr_full, pr_empty, pr_done;   // partner P: landed here / ours consumed there / our P.V of it done
    uint64_t mx_full[kMx], mx_empty[kMx], fin_full;
    float mx_in[kMx][kRows];               // the partner's block row maxima (log2 units)
    float fin_in[2][kRows];                // the partner's row sums (exact, bf16-rounded)
    uint32_t tmem_base;
    int dec[kDec];
    int abort;
};

constexpr int smem_bytes() {
    return kQSmemBytes + kSPartBytes + kNV * kVHalfBytes + 2 * kPBytes + (int)sizeof(Tail) + 1024;
}

__device__ __forceinline__ void set_timeout(Tail *t, unsigned int *status) {
    t->abort = 1;
    if (status) atomicOr(status, kStatusTimeout);
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    mla_pair_kernel(const MlaParams p, const __grid_constant__ CUtensorMap tmap_q,
                    const __grid_constant__ CUtensorMap tmap_k) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sq = smem;                                // Q boxes 6..8
    uint8_t *spart = sq + kQSmemBytes;                 // S-only boxes of an own block
    uint8_t *vring = spart + kSPartBytes;              // value boxes, every block
    uint8_t *pstage = vring + kNV * kVHalfBytes;       // own P (A operand here, source of the copy)
    uint8_t *pring = pstage + kPBytes;                 // the partner's P
    Tail *tl = reinterpret_cast<Tail *>(pring + kPBytes);

    const uint32_t h = cluster_ctarank();              // value columns 256h ..
    const uint32_t peer = h ^ 1u;
    const int split = blockIdx.x >> 1, b = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int j0 = split * p.per_split;
    const int j1 = min(p.nb, j0 + p.per_split);
    const int nblk = max(0, j1 - j0);

    if (threadIdx.x == 0) {
        mbar_init(&tl->q_full, 1);
        mbar_init(&tl->qt_full, 4);
        mbar_init(&tl->sp_full, 1);
        mbar_init(&tl->sp_empty, 1);
        for (int i = 0; i < kNV; i++) {
            mbar_init(&tl->v_full[i], 1);
            mbar_init(&tl->v_empty[i], 1);
        }
        mbar_init(&tl->s_full, 1);
        mbar_init(&tl->s_free, 4);
        mbar_init(&tl->o_done, 1);
        mbar_init(&tl->own_pv_done, 1);
        mbar_init(&tl->mma_done, 1);
        for (int i = 0; i < kDec; i++) {
            mbar_init(&tl->p_ready[i], 4);
            mbar_init(&tl->dec_free[i], 1);
        }
        mbar_init(&tl->pr_full, 1);
        mbar_init(&tl->pr_empty, 1);
        mbar_init(&tl->pr_done, 1);
        for (int i = 0; i < kMx; i++) {
            mbar_init(&tl->mx_full[i], 4);
            mbar_init(&tl->mx_empty[i], 4);
        }
        mbar_init(&tl->fin_full, 4);
        tl->abort = 0;
        fence_mbar_init();
    }
    if (warp == 5) {
        tmem_alloc(&tl->tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();  // both CTAs' barriers exist before either arrives on the other's
    tc_fence_after();
    const uint32_t tmem = tl->tmem_base;

    if (warp == 4) {
        // ------------------------------------------------------------------ producer
        if (lane == 0 && nblk > 0) {
            tma_prefetch_desc(&tmap_q);
            tma_prefetch_desc(&tmap_k);
            mbar_arrive_expect_tx(&tl->q_full, kQSmemBytes);
            for (int x = kQTmem; x < kBoxes; x++)
                tma_load_3d(sq + (x - kQTmem) * kQBoxBytes, &tmap_q, &tl->q_full, x * 64, 0, b);
            int v_issued = 0, sp_issued = 0;
            for (int jj = 0; jj < nblk && !tl->abort; jj++) {
                const int key0 = (j0 + jj) * kBN;
                const bool own = (uint32_t)(jj & 1) == h;
                if (own) {  // the 5 boxes only S reads: the other half's latent boxes, then RoPE
                    const int o = jj >> 1;
                    if (o >= 1 && !mbar_wait(&tl->sp_empty, (o - 1) & 1, &tl->abort)) {
                        set_timeout(tl, p.status);
                        break;
                    }
                    mbar_arrive_expect_tx(&tl->sp_full, kSPartBytes);
                    for (int i = 0; i < 4; i++)
                        tma_load_3d(spart + i * kKBoxBytes, &tmap_k, &tl->sp_full, (int)(4 * peer + i) * 64, key0, b);
                    tma_load_3d(spart + 4 * kKBoxBytes, &tmap_k, &tl->sp_full, 8 * 64, key0, b);
                    sp_issued++;
                }
                const int vs = jj % kNV;
                if (jj >= kNV && !mbar_wait(&tl->v_empty[vs], ((jj / kNV) & 1) ^ 1, &tl->abort)) {
                    set_timeout(tl, p.status);
                    break;
                }
                mbar_arrive_expect_tx(&tl->v_full[vs], kVHalfBytes);
                for (int i = 0; i < 4; i++)
                    tma_load_3d(vring + vs * kVHalfBytes + i * kKBoxBytes, &tmap_k, &tl->v_full[vs],
                                (int)(4 * h + i) * 64, key0, b);
                v_issued++;
            }
            mbar_wait(&tl->q_full, 0, nullptr);  // Q landed before this warp moves on
            if (tl->abort) {  // let copies already issued land
                if (sp_issued > 0) mbar_wait(&tl->sp_full, (sp_issued - 1) & 1, nullptr);
                for (int i = max(0, v_issued - kNV); i < v_issued; i++)
                    mbar_wait(&tl->v_full[i % kNV], (i / kNV) & 1, nullptr);
            }
        }
    } else if (warp == 5) {
        // --------------------------------------------------------------- MMA issuer
        if (lane == 0 && nblk > 0) {
            constexpr uint32_t idesc_s = umma_idesc_bf16(128, kBN, 0);
            constexpr uint32_t idesc_pv = umma_idesc_bf16(128, 256, 1);
            constexpr uint32_t dhi = umma_desc_hi_sw128();
            const uint32_t q_lo = umma_desc_lo(smem_addr(sq), 16);
            const uint32_t sp_lo = umma_desc_lo(smem_addr(spart), 16);
            const uint32_t v_lo = umma_desc_lo(smem_addr(vring), 16);          // K-major view (S)
            const uint32_t vmn_lo = umma_desc_lo(smem_addr(vring), kKBoxBytes);  // MN-major view (P.V)
            const uint32_t pst_lo = umma_desc_lo(smem_addr(pstage), 16);
            const uint32_t pr_lo = umma_desc_lo(smem_addr(pring), 16);
            const uint32_t s_col = tmem + kColS, q_col = tmem + kColQ, o_col = tmem + kColO;
            const uint32_t peer_pr_empty = mapa_shared(smem_addr(&tl->pr_empty), peer);
            bool ok = mbar_wait(&tl->q_full, 0, &tl->abort) && mbar_wait(&tl->qt_full, 0, &tl->abort);
            if (!ok) set_timeout(tl, p.status);
            // S = Q . K^T over the 576 columns in box order 0..8 (the order every pass of
            // this library uses, so that the scores are bit-identical across passes)
            auto issue_s = [&](int jj) {
                const uint32_t vst = v_lo + (uint32_t)(((jj % kNV) * kVHalfBytes) >> 4);
#pragma unroll
                for (int x = 0; x < kBoxes; x++) {
                    const int xi = x - 4 * (int)h;  // box index within this CTA's value boxes
                    const bool in_v = x < 8 && xi >= 0 && xi < 4;
                    const int si = x == 8 ? 4 : (x - 4 * (int)peer);  // index within the S-only stage
                    const uint32_t kb = in_v ? vst + (uint32_t)((xi * kKBoxBytes) >> 4)
                                             : sp_lo + (uint32_t)((si * kKBoxBytes) >> 4);
#pragma unroll
                    for (int kk = 0; kk < 4; kk++) {
                        const uint32_t kd = kb + (uint32_t)((kk * 32) >> 4);
                        if (x < kQTmem)
                            umma_ts2(s_col, q_col + (uint32_t)(x * 32 + kk * 8), kd, dhi, idesc_s, (x | kk) ? 1u : 0u);
                        else
                            umma_ss2(s_col, q_lo + (uint32_t)(((x - kQTmem) * kQBoxBytes + kk * 32) >> 4), kd, dhi,
                                     idesc_s, 1u);
                    }
                }
                umma_commit(&tl->s_full);
                umma_commit(&tl->sp_empty);  // the S-only boxes are free once S completes
            };
            int so = 0;                        // own S issued
            int jn = (int)h;                   // next own block
            int np = 0;                        // decisions taken
            int n_pv = 0, n_pr = 0, relays = 0;
            long long t_last = clock64();
            while (ok && (np < nblk || relays < n_pr)) {
                bool did = false;
                if (jn < nblk && mbar_test_wait(&tl->sp_full, so & 1) &&
                    mbar_test_wait(&tl->v_full[jn % kNV], (jn / kNV) & 1) &&
                    (so == 0 || mbar_test_wait(&tl->s_free, (so - 1) & 1))) {
                    tc_fence_after();
                    issue_s(jn);
                    so++;
                    jn += 2;
                    did = true;
                }
                if (np < nblk && mbar_test_wait(&tl->p_ready[np % kDec], (np / kDec) & 1)) {
                    const bool own = (uint32_t)(np & 1) == h;
                    const bool kept = tl->dec[np % kDec] != 0;
                    if (!kept || own || mbar_test_wait(&tl->pr_full, n_pr & 1)) {
                        tc_fence_after();
                        const int vs = np % kNV;
                        if (kept) {
                            const uint32_t a_lo = own ? pst_lo : pr_lo;
                            const uint32_t vst = vmn_lo + (uint32_t)((vs * kVHalfBytes) >> 4);
#pragma unroll
                            for (int kk = 0; kk < kBN / 16; kk++)
                                umma_ss2(o_col, a_lo + (uint32_t)((kk * 32) >> 4),
                                         vst + (uint32_t)((kk * 16 * 128) >> 4), dhi, idesc_pv,
                                         (n_pv > 0 || kk > 0) ? 1u : 0u);
                            umma_commit(&tl->o_done);
                            n_pv++;
                            if (own) {
                                umma_commit(&tl->own_pv_done);
                            } else {
                                umma_commit(&tl->pr_done);
                                n_pr++;
                            }
                        }
                        umma_commit(&tl->v_empty[vs]);
                        mbar_arrive(&tl->dec_free[np % kDec]);
                        np++;
                        did = true;
                    }
                }
                // the partner's P tile is free again once our P.V of it has completed
                if (relays < n_pr && mbar_test_wait(&tl->pr_done, relays & 1)) {
                    mbar_arrive_remote(peer_pr_empty);
                    relays++;
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
        // ------------------------------------------------------ softmax / decision
        const int row = threadIdx.x;  // 0..127, TMEM lane
        const bool valid_row = row < p.R;
        const int pos = row % p.Lq;
        const int last_key = !valid_row ? -1 : (p.causal ? pos + p.Lk - p.Lq : p.Lk - 1);
        const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
        const uint32_t s_addr = tmem + lane_off + kColS, o_addr = tmem + lane_off + kColO;
        {  // Q boxes 0..5 of this row -> TMEM, packed bf16 pairs
            const uint16_t *qrow = p.q + ((size_t)b * p.R + (valid_row ? row : 0)) * 576;
#pragma unroll 1
            for (int x = 0; x < kQTmem; x++) {
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
        const uint32_t peer_mx_in = mapa_shared(smem_addr(&tl->mx_in[0][row]), peer);
        const uint32_t peer_mx_full = mapa_shared(smem_addr(&tl->mx_full[0]), peer);
        const uint32_t peer_mx_empty = mapa_shared(smem_addr(&tl->mx_empty[0]), peer);
        const uint32_t peer_pr_full = mapa_shared(smem_addr(&tl->pr_full), peer);
        const uint32_t peer_pring = mapa_shared(smem_addr(pring), peer);
        const float NEG_INF = -CUDART_INF_F;
        const bool report = h == 0;  // one CTA of the pair writes mask and count
        float m_true = NEG_INF, m_ref = NEG_INF, l = 0.f, lr = 0.f;
        int n_kept = 0, n_own_p = 0;
        unsigned int n_skip = 0;
        uint32_t mword = 0;
        int mword_idx = -1;
        // An own block's scores come out of tensor memory, and its row maxima go to the
        // partner, one block AHEAD of its decision: while waiting for the maxima of the
        // partner's block in front of it.  The two CTAs therefore never wait on each
        // other's decisions to send their own maxima.
        float s[64];    // scores of the next own block (log2 units after scaling in the exp)
        float mt_own = NEG_INF;
        int n_read = 0;  // own blocks read so far
        auto read_own = [&](int jo) {  // S of own block jo -> s[], row max -> partner
            const int o = jo >> 1;
            if (!mbar_wait(&tl->s_full, o & 1, &tl->abort)) set_timeout(tl, p.status);
            tc_fence_after();
            {
                uint32_t *sr = reinterpret_cast<uint32_t *>(s);
                tmem_ld32(s_addr, sr);
                tmem_ld32(s_addr + 32, sr + 32);
                tc_wait_ld();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tl->s_free);  // the next own S may overwrite it now
            const int lim = last_key - (j0 + jo) * kBN;
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
            mt_own = fmax3(m0, m1, fmaxf(m2, m3)) * p.scale_log2;
            const int slot = o % kMx;
            if (o >= kMx && !mbar_wait_cluster(&tl->mx_empty[slot], ((o / kMx) - 1) & 1, &tl->abort))
                set_timeout(tl, p.status);
            st_cluster_f32(peer_mx_in + (uint32_t)(slot * kRows * 4), mt_own);
            fence_acq_rel_cluster();
            __syncwarp();
            if (lane == 0) mbar_arrive_remote(peer_mx_full + (uint32_t)(slot * 8));
            n_read++;
        };
        for (int jj = 0; jj < nblk; jj++) {
            const int j = j0 + jj;
            const bool own = (uint32_t)(jj & 1) == h;
            const int o = jj >> 1;  // index among the owner's blocks
            float mt;
            if (own) {
                if (n_read <= o) read_own(jj);  // (only the first own block of CTA 0 is read here)
                mt = mt_own;
            } else {
                if (jj + 1 < nblk) read_own(jj + 1);  // the next block is ours: read and send it first
                const int slot = o % kMx;
                if (!mbar_wait_cluster(&tl->mx_full[slot], (o / kMx) & 1, &tl->abort)) set_timeout(tl, p.status);
                mt = tl->mx_in[slot][row];
                __syncwarp();
                if (lane == 0) mbar_arrive_remote(peer_mx_empty + (uint32_t)(slot * 8));
            }
            const float mn = fmaxf(m_true, mt);
            const bool vote = (mt == NEG_INF) || (mt - mn < p.thr_log2);
            // (every block below Lk is visited: the last query row sees all keys)
            const bool all = bar_and(1, 128, vote);
            const bool skip = all && jj > 0;
            const bool kept = !skip;
            // at most kDec decisions outstanding at the MMA thread
            if (jj >= kDec && !mbar_wait(&tl->dec_free[jj % kDec], ((jj / kDec) - 1) & 1, &tl->abort))
                set_timeout(tl, p.status);
            if (row == 0) tl->dec[jj % kDec] = kept ? 1 : 0;
            if (kept) {
                m_true = mn;
                const bool warp_need = __any_sync(0xffffffffu, mn - m_ref > kRescaleThreshold);
                float alpha = 1.f;
                if (warp_need) {
                    alpha = (m_ref == NEG_INF || mn == NEG_INF) ? (mn == NEG_INF ? 1.f : 0.f) : ex2(m_ref - mn);
                    l *= alpha;
                    lr *= alpha;
                    if (mn != NEG_INF) m_ref = mn;
                    if (n_kept > 0) {  // every earlier P.V has landed before O is rescaled
                        if (!mbar_wait(&tl->o_done, (n_kept - 1) & 1, &tl->abort)) set_timeout(tl, p.status);
                        tc_fence_after();
#pragma unroll 1
                        for (int c = 0; c < 8; c++) {
                            uint32_t orr[32];
                            tmem_ld32(o_addr + c * 32, orr);
                            tc_wait_ld();
#pragma unroll
                            for (int i = 0; i < 32; i++) orr[i] = __float_as_uint(__uint_as_float(orr[i]) * alpha);
                            tmem_st32(o_addr + c * 32, orr);
                        }
                        tc_wait_st();
                    }
                }
                if (own) {
                    // the staging tile is free once our last P.V from it and the partner's
                    // P.V from its copy have completed
                    if (n_own_p > 0) {
                        if (!mbar_wait(&tl->own_pv_done, (n_own_p - 1) & 1, &tl->abort) ||
                            !mbar_wait(&tl->pr_empty, (n_own_p - 1) & 1, &tl->abort))
                            set_timeout(tl, p.status);
                    }
                    const float mref = m_ref == NEG_INF ? 0.f : m_ref;
                    float rs = 0.f, rr = 0.f;
                    uint8_t *prow = pstage + row * 128;
#pragma unroll
                    for (int c = 0; c < 8; c++) {  // keys 8c .. 8c+7 -> 16-byte chunk c (128-byte swizzle)
                        uint32_t pk[4];
#pragma unroll
                        for (int u = 0; u < 4; u++) {
                            const float p0 = ex2(fmaf(s[8 * c + 2 * u], p.scale_log2, -mref));
                            const float p1 = ex2(fmaf(s[8 * c + 2 * u + 1], p.scale_log2, -mref));
                            pk[u] = pack_bf16x2(p0, p1);
                            rs += p0 + p1;
                            rr += __uint_as_float(pk[u] << 16) + __uint_as_float(pk[u] & 0xFFFF0000u);
                        }
                        *reinterpret_cast<uint4 *>(prow + ((c ^ (row & 7)) << 4)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                    }
                    l += rs;
                    lr += rr;
                    fence_proxy_async();  // the tile is read by the tensor cores and the bulk copy
                    bar_sync(2, 128);
                    if (row == 0) {
                        mbar_arrive_expect_tx_remote(peer_pr_full, kPBytes);
                        bulk_copy_to_peer(peer_pring, pstage, kPBytes, peer_pr_full);
                    }
                    n_own_p++;
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&tl->p_ready[jj % kDec]);
                n_kept++;
            } else {
                __syncwarp();
                if (lane == 0) mbar_arrive(&tl->p_ready[jj % kDec]);
                n_skip++;
                if (row == 0 && report && p.skip_mask) {
                    if (mword_idx != (j >> 5)) {
                        if (mword_idx >= 0 && mword) atomicOr(p.skip_mask + (size_t)b * p.words + mword_idx, mword);
                        mword_idx = j >> 5;
                        mword = 0;
                    }
                    mword |= 1u << (j & 31);
                }
            }
        }
        if (row == 0 && report) {
            if (p.skip_mask && mword_idx >= 0 && mword) atomicOr(p.skip_mask + (size_t)b * p.words + mword_idx, mword);
            if (p.skip_count && n_skip) atomicAdd(p.skip_count, (unsigned long long)n_skip);
        }
        // our last P reached the partner and was used there before this CTA may finish
        if (n_own_p > 0 && !mbar_wait(&tl->pr_empty, (n_own_p - 1) & 1, &tl->abort)) set_timeout(tl, p.status);
        // row sums: ours cover our own blocks; add the partner's
        st_cluster_f32(mapa_shared(smem_addr(&tl->fin_in[0][row]), peer), l);
        st_cluster_f32(mapa_shared(smem_addr(&tl->fin_in[1][row]), peer), lr);
        fence_acq_rel_cluster();
        __syncwarp();
        if (lane == 0) mbar_arrive_remote(mapa_shared(smem_addr(&tl->fin_full), peer));
        if (!mbar_wait_cluster(&tl->fin_full, 0, &tl->abort)) set_timeout(tl, p.status);
        const float l_tot = l + tl->fin_in[0][row];
        const float lr_tot = lr + tl->fin_in[1][row];
        // split epilogue: normalised partial O (this CTA's 256 value columns), the split's lse
        const size_t orow = ((size_t)b * p.R + row) * p.num_splits + split;
        if (n_kept > 0) {
            if (!mbar_wait(&tl->o_done, (n_kept - 1) & 1, &tl->abort)) set_timeout(tl, p.status);
            tc_fence_after();
        }
        const float inv = lr_tot > 0.f ? 1.f / lr_tot : 0.f;
#pragma unroll 1
        for (int c = 0; c < 8; c++) {
            uint32_t orr[32];
            tmem_ld32(o_addr + c * 32, orr);
            tc_wait_ld();
            if (valid_row) {
                float *dst = p.part_o + orow * 512 + h * 256 + c * 32;
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
        if (valid_row && h == 0)
            p.part_lse[orow] = l_tot > 0.f ? (m_ref + __log2f(l_tot)) * 0.69314718055994531f : NEG_INF;
    } else if (warp < 4) {
        // an empty split: its partial output is empty (lse = -inf) and the combine ignores it
        const int row = threadIdx.x;
        if (row < p.R) {
            const size_t orow = ((size_t)b * p.R + row) * p.num_splits + split;
            float *dst = p.part_o + orow * 512 + h * 256;
            for (int i = 0; i < 256; i += 4) *reinterpret_cast<float4 *>(dst + i) = make_float4(0.f, 0.f, 0.f, 0.f);
            if (h == 0) p.part_lse[orow] = -CUDART_INF_F;
        }
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();  // no remote access to this CTA's shared memory is left in flight
    tc_fence_after();
    if (warp == 5) tmem_dealloc(tmem, 512);
}

}  // namespace pair

}  // namespace

cudaError_t launch_mla(const MlaParams &p, const CUtensorMap &tq, const CUtensorMap &tk, bool calib,
                       cudaStream_t st) {
    if (calib) {
        constexpr int smem = calib::smem_bytes();
        cudaError_t e = cudaFuncSetAttribute(calib::mla_calib_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        dim3 grid(p.num_splits, 1, p.B);
        calib::mla_calib_kernel<<<grid, calib::kThreads, smem, st>>>(p, tq, tk);
        return cudaGetLastError();
    }
    constexpr int smem = pair::smem_bytes();
    cudaError_t e = cudaFuncSetAttribute(pair::mla_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    dim3 grid(2 * p.num_splits, 1, p.B);
    pair::mla_pair_kernel<<<grid, pair::kThreads, smem, st>>>(p, tq, tk);
    return cudaGetLastError();
}

}  // namespace blasst
