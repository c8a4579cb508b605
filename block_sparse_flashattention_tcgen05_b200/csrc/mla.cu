// mla.cu -- split-KV MLA decode with softmax-threshold block skipping (BLASST)
// on tcgen05: one latent KV head of 576 columns (512 latent + 64 RoPE) shared
// by every query head; Q.K^T contracts all 576 columns, P.V uses the first
// 512 columns of the same cache rows as V.
//
// A cluster of two CTAs handles one (split, sequence).  The tile is all
// G = Hq query heads x Lq queries (G*Lq <= 128 rows, one TMEM lane each); KV
// blocks of 64 keys.  The 128 x 512 fp32 output does not fit one SM's tensor
// memory next to S, so the two CTAs split the columns:
//   rank 0 holds latent columns 0..255 and the 64 RoPE columns,
//   rank 1 holds latent columns 256..511,
// of both Q and each K block.  Each CTA computes a partial S over its columns
// and copies it (fp32) into the other CTA's shared memory; both form
// S = S0 + S1 in the same order, so both take the same skip decision, and each
// accumulates P.V for the 256 value columns it already holds.  Neither the
// Q.K^T products nor the K bytes are duplicated.
//
// The exchange: rows are written to a local staging buffer and one thread copies
// the 32 KB partial into the peer's receive buffer with a bulk shared-to-shared
// copy; the peer's arrive on recv_free returns both buffers for the next block.
//
// Warp roles (192 threads per CTA): warps 0-3 softmax/decision (thread = row),
// warp 4 TMA producer (own Q columns once, own K columns per block into a
// 2-stage ring), warp 5 TMEM allocation + tcgen05.mma issue.
// TMEM: S_part [0,64), P double buffer [64,96) [96,128) (bf16), O_half [256,512).
//
// Per block: partial S (always), exchange, tile decision as in the other
// kernels (true running max, restarted per split, first visited block kept);
// kept blocks: lazy O rescale, P = 2^(s - M_ref) -> bf16 in TMEM, O += P V_j.
// Skipped blocks skip exp and P.V; their V bytes are K bytes already loaded
// (V adds no memory traffic in MLA).
#include <cuda_bf16.h>
#include <math_constants.h>

#include "internal.h"
#include "ptx.cuh"

namespace blasst {
namespace {

constexpr int kThreads = 192;
constexpr int kRows = 128;
constexpr int kBN = 64;
constexpr int kMaxBoxes = 5;                          // 64-column boxes held by rank 0
constexpr int kQBoxBytes = kRows * 128;               // 128 rows x 64 bf16
constexpr int kKBoxBytes = kBN * 128;                 // 64 keys x 64 bf16
constexpr int kStages = 2;
constexpr int kQBytes = kMaxBoxes * kQBoxBytes;       // 80 KB
constexpr int kKStageBytes = kMaxBoxes * kKBoxBytes;  // 40 KB
constexpr int kRecvBytes = kRows * kBN * 4;           // 32 KB: one partial S (staging and receive buffers)
constexpr float kRescaleThreshold = 8.0f;
constexpr int kStatusTimeout = 1;

struct MlaSmemTail {
    uint64_t q_full, k_full[kStages], k_empty[kStages], s_full, s_free, p_full, o_done, mma_done;
    uint64_t recv_full, recv_free;
    uint32_t tmem_base;
    int dec;
    int abort;
    float gred[4];
};

constexpr int mla_smem_bytes() {
    return kQBytes + kStages * kKStageBytes + 2 * kRecvBytes + (int)sizeof(MlaSmemTail) + 1024;
}

__device__ __forceinline__ void set_timeout(MlaSmemTail *t, unsigned int *status) {
    t->abort = 1;
    if (status) atomicOr(status, kStatusTimeout);
}

// Global 64-column box index of local slot `slot` on cluster rank `rank`.
__device__ __forceinline__ int box_of(uint32_t rank, int slot) {
    return rank == 0 ? (slot < 4 ? slot : 8) : 4 + slot;
}

template <bool CALIB>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    mla_split_kernel(const MlaParams p, const __grid_constant__ CUtensorMap tmap_q,
                     const __grid_constant__ CUtensorMap tmap_k) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sq = smem;
    uint8_t *sk = smem + kQBytes;
    uint8_t *srecv = sk + kStages * kKStageBytes;
    MlaSmemTail *tl = reinterpret_cast<MlaSmemTail *>(srecv + 2 * kRecvBytes);

    const uint32_t rank = cluster_ctarank();
    const uint32_t peer = rank ^ 1u;
    const int split = blockIdx.x >> 1, b = blockIdx.z;
    const int nbox = rank == 0 ? 5 : 4;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int j0 = split * p.per_split;
    const int j1 = min(p.nb, j0 + p.per_split);
    const int nblk = max(0, j1 - j0);

    if (threadIdx.x == 0) {
        mbar_init(&tl->q_full, 1);
        for (int i = 0; i < kStages; i++) {
            mbar_init(&tl->k_full[i], 1);
            mbar_init(&tl->k_empty[i], 1);
        }
        mbar_init(&tl->s_full, 1);
        mbar_init(&tl->s_free, 4);
        mbar_init(&tl->p_full, 4);
        mbar_init(&tl->o_done, 1);
        mbar_init(&tl->mma_done, 1);
        mbar_init(&tl->recv_full, 1);
        mbar_init(&tl->recv_free, 1);
        tl->abort = 0;
        fence_mbar_init();
        // the first exchange is armed before the peer can send
        if (nblk > 0) mbar_arrive_expect_tx(&tl->recv_full, kRecvBytes);
    }
    if (warp == 5) {
        tmem_alloc(&tl->tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    cluster_sync();  // both CTAs' barriers exist before any cross-CTA store
    const uint32_t tmem = tl->tmem_base;

    if (warp == 4) {
        // ---------------------------------------------------------------- producer
        if (lane == 0 && nblk > 0) {
            tma_prefetch_desc(&tmap_q);
            tma_prefetch_desc(&tmap_k);
            mbar_arrive_expect_tx(&tl->q_full, nbox * kQBoxBytes);
            for (int x = 0; x < nbox; x++)
                tma_load_3d(sq + x * kQBoxBytes, &tmap_q, &tl->q_full, box_of(rank, x) * 64, 0, b);
            int issued = 0;
            for (int jj = 0; jj < nblk && !tl->abort; jj++) {
                const int st = jj & 1;
                if (jj >= kStages && !mbar_wait(&tl->k_empty[st], ((jj >> 1) & 1) ^ 1, &tl->abort)) {
                    set_timeout(tl, p.status);
                    break;
                }
                mbar_arrive_expect_tx(&tl->k_full[st], nbox * kKBoxBytes);
                for (int x = 0; x < nbox; x++)
                    tma_load_3d(sk + st * kKStageBytes + x * kKBoxBytes, &tmap_k, &tl->k_full[st], box_of(rank, x) * 64,
                                (j0 + jj) * kBN, b);
                issued++;
            }
            if (tl->abort) {
                for (int jj = max(0, issued - kStages); jj < issued; jj++)
                    mbar_wait(&tl->k_full[jj & 1], (jj >> 1) & 1, nullptr);
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
            // V = this CTA's 256 latent columns = local slots 0..3 of the K stage, MN-major
            const uint32_t v_lo = umma_desc_lo(smem_addr(sk), kKBoxBytes);
            const uint32_t s_col = tmem, o_col = tmem + 256;
            bool ok = mbar_wait(&tl->q_full, 0, &tl->abort);
            auto issue_s = [&](int jj) {
                const uint32_t kst = k_lo + (uint32_t)((jj & 1) * kKStageBytes >> 4);
                for (int x = 0; x < nbox; x++)
#pragma unroll
                    for (int kk = 0; kk < 4; kk++)
                        umma_ss2(s_col, q_lo + (uint32_t)((x * kQBoxBytes + kk * 32) >> 4),
                                 kst + (uint32_t)((x * kKBoxBytes + kk * 32) >> 4), dhi, idesc_s, (x | kk) ? 1u : 0u);
                umma_commit(&tl->s_full);
            };
            if (ok && !mbar_wait(&tl->k_full[0], 0, &tl->abort)) ok = false;
            if (ok) {
                tc_fence_after();
                issue_s(0);
            }
            int n_pv = 0;
            for (int jj = 0; jj < nblk && ok; jj++) {
                if (jj + 1 < nblk) {
                    // S(jj+1) overwrites S(jj) once the softmax holds it in registers
                    if (!mbar_wait(&tl->s_free, jj & 1, &tl->abort) ||
                        !mbar_wait(&tl->k_full[(jj + 1) & 1], ((jj + 1) >> 1) & 1, &tl->abort)) {
                        set_timeout(tl, p.status);
                        break;
                    }
                    tc_fence_after();
                    issue_s(jj + 1);
                }
                if (!mbar_wait(&tl->p_full, jj & 1, &tl->abort)) {
                    set_timeout(tl, p.status);
                    break;
                }
                tc_fence_after();
                if (!CALIB && tl->dec) {
                    const uint32_t p_col = tmem + 64 + (uint32_t)(jj & 1) * 32;
                    const uint32_t vst = v_lo + (uint32_t)((jj & 1) * kKStageBytes >> 4);
#pragma unroll
                    for (int kk = 0; kk < kBN / 16; kk++)
                        umma_ts2(o_col, p_col + kk * 8, vst + (uint32_t)((kk * 16 * 128) >> 4), dhi, idesc_pv,
                                 (n_pv > 0 || kk > 0) ? 1u : 0u);
                    umma_commit(&tl->o_done);
                    n_pv++;
                }
                umma_commit(&tl->k_empty[jj & 1]);
            }
            umma_commit(&tl->mma_done);
            if (!mbar_wait(&tl->mma_done, 0, nullptr)) set_timeout(tl, p.status);
        }
        __syncwarp();
    } else {
        // ----------------------------------------------------- softmax / decision
        const int row = threadIdx.x;  // 0..127, TMEM lane
        const bool valid_row = row < p.R;
        const int pos = row % p.Lq;
        const int last_key = !valid_row ? -1 : (p.causal ? pos + p.Lk - p.Lq : p.Lk - 1);
        const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
        const uint32_t s_addr = tmem + lane_off, o_addr = tmem + lane_off + 256;
        uint8_t *stage = srecv;               // my partial, copied to the peer
        uint8_t *recv = srecv + kRecvBytes;   // the peer's partial
        const uint32_t recv_remote = mapa_shared(smem_addr(recv), peer);
        const uint32_t recv_full_remote = mapa_shared(smem_addr(&tl->recv_full), peer);
        const uint32_t recv_free_remote = mapa_shared(smem_addr(&tl->recv_free), peer);
        const float NEG_INF = -CUDART_INF_F;
        float m_true = NEG_INF, m_ref = NEG_INF, l = 0.f, lr = 0.f;
        int n_kept = 0;
        bool seen = false;
        unsigned int n_skip = 0;
        uint32_t mword = 0;
        int mword_idx = -1;
        for (int jj = 0; jj < nblk; jj++) {
            const int j = j0 + jj;
            if (!mbar_wait(&tl->s_full, jj & 1, &tl->abort)) set_timeout(tl, p.status);
            tc_fence_after();
            uint32_t sr[64];
            tmem_ld32(s_addr, sr);
            tmem_ld32(s_addr + 32, sr + 32);
            tc_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tl->s_free);
            // exchange partial scores with the other CTA (rows swizzled by 16-byte chunk)
            if (jj > 0 && !mbar_wait_cluster(&tl->recv_free, (jj - 1) & 1, &tl->abort)) set_timeout(tl, p.status);
#pragma unroll
            for (int c = 0; c < 16; c++)
                *reinterpret_cast<uint4 *>(stage + row * 256 + ((c ^ (row & 15)) << 4)) =
                    make_uint4(sr[4 * c], sr[4 * c + 1], sr[4 * c + 2], sr[4 * c + 3]);
            fence_proxy_async();
            bar_sync(1, 128);
            if (row == 0) bulk_copy_to_peer(recv_remote, smem_addr(stage), kRecvBytes, recv_full_remote);
            if (!mbar_wait_cluster(&tl->recv_full, jj & 1, &tl->abort)) set_timeout(tl, p.status);
            float s[64];
#pragma unroll
            for (int c = 0; c < 16; c++) {
                const float4 v = *reinterpret_cast<const float4 *>(recv + row * 256 + ((c ^ (row & 15)) << 4));
                const float o0 = __uint_as_float(sr[4 * c]), o1 = __uint_as_float(sr[4 * c + 1]);
                const float o2 = __uint_as_float(sr[4 * c + 2]), o3 = __uint_as_float(sr[4 * c + 3]);
                // S = S0 + S1 in the same order on both CTAs
                s[4 * c] = rank == 0 ? o0 + v.x : v.x + o0;
                s[4 * c + 1] = rank == 0 ? o1 + v.y : v.y + o1;
                s[4 * c + 2] = rank == 0 ? o2 + v.z : v.z + o2;
                s[4 * c + 3] = rank == 0 ? o3 + v.w : v.w + o3;
            }
            // every row has read the peer's partial: re-arm for the next block, then
            // tell the peer that its staging and this receive buffer are free again
            bar_sync(1, 128);
            if (row == 0) {
                if (jj + 1 < nblk) mbar_arrive_expect_tx(&tl->recv_full, kRecvBytes);
                mbar_arrive_remote(recv_free_remote);
            }

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
            const bool all = bar_and(1, 128, vote);
            const bool visited = !bar_and(1, 128, mt == NEG_INF);
            const bool first = visited && !seen;
            seen = seen || visited;
            const bool skip = visited && all && !first;
            const bool kept = visited && !skip;
            if (CALIB && rank == 0 && p.gaps) {
                float g = mt == NEG_INF ? NEG_INF : mt - mn;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) g = fmaxf(g, __shfl_xor_sync(0xffffffffu, g, o));
                if (lane == 0) tl->gred[warp] = g;
                bar_sync(1, 128);
                if (row == 0) {
                    const float gg = fmaxf(fmaxf(tl->gred[0], tl->gred[1]), fmaxf(tl->gred[2], tl->gred[3]));
                    p.gaps[(size_t)b * p.nb + j] =
                        !visited ? CUDART_NAN_F : (first ? CUDART_INF_F : gg * 0.69314718055994531f);
                }
                bar_sync(1, 128);
            }
            if (row == 0) tl->dec = kept ? 1 : 0;
            if (!kept || CALIB) {
                if (kept) m_true = mn;
                __syncwarp();
                if (lane == 0) mbar_arrive(&tl->p_full);
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
                const uint32_t p_addr = tmem + lane_off + 64 + (uint32_t)(jj & 1) * 32;
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
                }
                tc_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&tl->p_full);
                n_kept++;
            }
            if (skip) n_skip++;
            if (row == 0 && rank == 0 && p.skip_mask && skip) {
                if (mword_idx != (j >> 5)) {
                    if (mword_idx >= 0 && mword) atomicOr(p.skip_mask + (size_t)b * p.words + mword_idx, mword);
                    mword_idx = j >> 5;
                    mword = 0;
                }
                mword |= 1u << (j & 31);
            }
        }
        if (row == 0 && rank == 0) {
            if (p.skip_mask && mword_idx >= 0 && mword) atomicOr(p.skip_mask + (size_t)b * p.words + mword_idx, mword);
            if (p.skip_count && n_skip) atomicAdd(p.skip_count, (unsigned long long)n_skip);
        }
        if (!CALIB) {
            // split epilogue: normalised partial O (this CTA's 256 value columns), the split's lse
            const size_t orow = ((size_t)b * p.R + row) * p.num_splits + split;
            if (n_kept > 0) {
                if (!mbar_wait(&tl->o_done, (n_kept - 1) & 1, &tl->abort)) set_timeout(tl, p.status);
                tc_fence_after();
            }
            const float inv = lr > 0.f ? 1.f / lr : 0.f;
#pragma unroll 1
            for (int c = 0; c < 8; c++) {
                uint32_t orr[32];
                tmem_ld32(o_addr + c * 32, orr);
                tc_wait_ld();
                if (valid_row) {
                    float *dst = p.part_o + orow * 512 + rank * 256 + c * 32;
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
            if (valid_row && rank == 0)
                p.part_lse[orow] = l > 0.f ? (m_ref + __log2f(l)) * 0.69314718055994531f : NEG_INF;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 5) tmem_dealloc(tmem, 512);
    cluster_sync();  // no CTA leaves while its peer may still address its shared memory
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
