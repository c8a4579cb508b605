// decode_wide.cu -- split-KV decode with softmax-threshold block skipping (BLASST)
// for wide query tiles on tcgen05: the G query heads x Lq queries that share a KV
// head, 17 to 128 rows (MQA with many heads, GQA with large groups), d = dv = 128.
// Narrower tiles take the mma.sync kernel in decode.cu.
//
// One CTA per (split, KV head, sequence).  Rows of the tile are TMEM lanes; KV
// blocks of 64 keys.  Per block: S = Q K_j^T (M = 128, N = 64, K = 128) into TMEM,
// block row maxima, the true running max (restarted per split), the tile-wide
// skip vote (first block of a split kept) -- all before any V traffic: a V producer
// warp loads V_j only for kept blocks (xllm-io paper review, section 3, decode
// kernel optimisation: V of pruned blocks is never loaded).  Kept blocks: lazy O
// rescale, P = 2^(s - M_ref) in TMEM, O += P V_j (M = 128, N = 128, K = 64).
//
// Warp roles (224 threads): warps 0-3 softmax/decision (thread = row), warp 4 TMA
// producer of Q (once) and K (2-stage ring), warp 5 TMEM allocation + tcgen05.mma
// issue, warp 6 V producer (2-stage ring, kept blocks only).  Two CTAs share an SM
// (99 KB of shared memory and 256 TMEM columns each).
// TMEM (256 columns): S [0,64), P [64,128) as two bf16 buffers, O [128,256).
// A K stage goes back to its producer as soon as S has read it, and kept blocks
// alternate between the two P buffers, so the softmax writes P(k) once the P.V of
// kept block k-2 (not k-1) is done: two V loads stay in flight behind the
// decisions instead of one.
// Seeded splits: every split after the first scores block 0 ahead of its own
// blocks; that block's row maxima start the split's running max (no decision,
// no exp, no P.V, nothing reported), and the split has no forced first block.
#include <cuda_bf16.h>
#include <math_constants.h>

#include "internal.h"
#include "ptx.cuh"

namespace blasst {
namespace {

constexpr int kThreads = 224;
constexpr int kRows = 128;
constexpr int kBN = kDecodeBlockN;
constexpr int kBoxBytesQ = kRows * 128;    // 128 rows x 64 bf16
constexpr int kBoxBytesKV = kBN * 128;     // 64 keys x 64 bf16
constexpr int kStageBytes = 2 * kBoxBytesKV;
constexpr int kQBytes = 2 * kBoxBytesQ;
constexpr int kNK = 2, kNV = 2;   // two CTAs per SM: each keeps two blocks of K and of V in flight
constexpr int kMaxWideBlocks = 1024;  // ring entries per split, seed block included (decision array)
constexpr uint32_t kColP = 64, kColO = 128;  // P buffer b at kColP + 32 b
constexpr int kDecRing = 8;                    // decisions published ahead of the MMA thread
constexpr float kRescaleThreshold = 8.0f;
constexpr int kStatusTimeout = 1;
constexpr int kStatusBadPage = 2;

struct WideSmemTail {
    uint64_t q_full, k_full[kNK], k_empty[kNK], v_full[kNV], v_empty[kNV];
    uint64_t s_full, s_free, mma_done;
    uint64_t o_done[2];  // [P buffer]: the P.V that read it has completed
    uint64_t p_full[kDecRing], dec_free[kDecRing];  // block decisions (and P) ready / taken
    uint32_t tmem_base;
    int dec_count;       // decisions published (blocks of this split)
    int abort;
    float gred[4];
};

constexpr int wide_smem_bytes(bool calib) {
    return kQBytes + kNK * kStageBytes + (calib ? 0 : kNV * kStageBytes) + (int)sizeof(WideSmemTail) +
           kMaxWideBlocks + 1024;
}

__device__ __forceinline__ void set_timeout(WideSmemTail *t, unsigned int *status) {
    t->abort = 1;
    if (status) atomicOr(status, kStatusTimeout);
}

// TMA coordinates (row, plane) of block blk of KV head hkv of sequence b (paged or not).
__device__ __forceinline__ int2 block_coord(const DecodeParams &p, int b, int hkv, int blk) {
    if (!p.block_table) return make_int2(blk * kBN, b * p.Hkv + hkv);
    int page = __ldg(p.block_table + (size_t)b * p.nb + blk);
    if (page < 0 || page >= p.num_pages) {
        if (p.status) atomicOr(p.status, kStatusBadPage);
        page = p.num_pages;
    }
    return make_int2(0, page * p.Hkv + hkv);
}

template <bool CALIB>
__global__ void __launch_bounds__(kThreads, 2)
    decode_wide_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap tmap_q,
                       const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sq = smem;
    uint8_t *sk = sq + kQBytes;
    uint8_t *sv = sk + kNK * kStageBytes;
    WideSmemTail *tl = reinterpret_cast<WideSmemTail *>(sv + (CALIB ? 0 : kNV * kStageBytes));
    volatile uint8_t *dec = reinterpret_cast<volatile uint8_t *>(tl + 1);

    const int split = blockIdx.x, hkv = blockIdx.y, b = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int Lk = p.Lk, nbs = p.nb, per_split = p.per_split;
    if (p.seq_lens) {
        Lk = __ldg(p.seq_lens + b);
        if (Lk < 0 || Lk > p.Lk) {
            if (threadIdx.x == 0 && p.status) atomicOr(p.status, kStatusBadPage);
            Lk = min(max(Lk, 0), p.Lk);
        }
        nbs = (Lk + kBN - 1) / kBN;
        per_split = (nbs + p.num_splits - 1) / p.num_splits;
    }
    const int j0 = split * per_split;
    const int j1 = min(nbs, j0 + per_split);
    const int nblk = max(0, j1 - j0);
    const int bh = b * p.Hkv + hkv;
    // ring entries: [block 0 (seed)], then the split's blocks j0 .. j1-1
    const int seed = (p.seed && split > 0 && nblk > 0) ? 1 : 0;
    const int nent = nblk + seed;
    auto entry_block = [&](int e) { return (seed && e == 0) ? 0 : j0 + e - seed; };

    if (threadIdx.x == 0) {
        mbar_init(&tl->q_full, 1);
        for (int i = 0; i < kNK; i++) {
            mbar_init(&tl->k_full[i], 1);
            mbar_init(&tl->k_empty[i], 1);
        }
        for (int i = 0; i < kNV; i++) {
            mbar_init(&tl->v_full[i], 1);
            mbar_init(&tl->v_empty[i], 1);
        }
        mbar_init(&tl->s_full, 1);
        mbar_init(&tl->s_free, 4);
        mbar_init(&tl->o_done[0], 1);
        mbar_init(&tl->o_done[1], 1);
        mbar_init(&tl->mma_done, 1);
        for (int i = 0; i < kDecRing; i++) {
            mbar_init(&tl->p_full[i], 4);
            mbar_init(&tl->dec_free[i], 1);
        }
        tl->dec_count = 0;
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
        // ---------------------------------------------------------- Q and K producer
        if (lane == 0 && nblk > 0) {
            tma_prefetch_desc(&tmap_q);
            tma_prefetch_desc(&tmap_k);
            const int qrow = hkv * p.G * p.Lq;  // the tile's first row within the sequence's Hq*Lq rows
            mbar_arrive_expect_tx(&tl->q_full, kQBytes);
            tma_load_3d(sq, &tmap_q, &tl->q_full, 0, qrow, b);
            tma_load_3d(sq + kBoxBytesQ, &tmap_q, &tl->q_full, 64, qrow, b);
            int issued = 0;
            for (int jj = 0; jj < nent && !tl->abort; jj++) {
                const int st = jj % kNK;
                if (jj >= kNK && !mbar_wait(&tl->k_empty[st], ((jj / kNK) & 1) ^ 1, &tl->abort)) {
                    set_timeout(tl, p.status);
                    break;
                }
                const int2 cr = block_coord(p, b, hkv, entry_block(jj));
                mbar_arrive_expect_tx(&tl->k_full[st], kStageBytes);
                tma_load_3d(sk + st * kStageBytes, &tmap_k, &tl->k_full[st], 0, cr.x, cr.y);
                tma_load_3d(sk + st * kStageBytes + kBoxBytesKV, &tmap_k, &tl->k_full[st], 64, cr.x, cr.y);
                issued++;
            }
            mbar_wait(&tl->q_full, 0, nullptr);
            for (int jj = max(0, issued - kNK); jj < issued; jj++)  // copies in flight land before exit
                mbar_wait(&tl->k_full[jj % kNK], (jj / kNK) & 1, nullptr);
        }
    } else if (warp == 6) {
        // ------------------------------------------------- V producer (kept blocks)
        if (!CALIB && lane == 0 && nblk > 0) {
            tma_prefetch_desc(&tmap_v);
            int vk = 0;
            for (int jj = 0; jj < nent && !tl->abort; jj++) {
                long long t0 = clock64();
                while (*reinterpret_cast<volatile int *>(&tl->dec_count) <= jj) {
                    if (tl->abort || clock64() - t0 > kWaitLimitCycles) {
                        set_timeout(tl, p.status);
                        break;
                    }
                    __nanosleep(64);
                }
                if (tl->abort) break;
                __threadfence_block();
                if (!dec[jj]) continue;
                const int st = vk % kNV;
                if (vk >= kNV && !mbar_wait(&tl->v_empty[st], ((vk / kNV) & 1) ^ 1, &tl->abort)) {
                    set_timeout(tl, p.status);
                    break;
                }
                const int2 cr = block_coord(p, b, hkv, entry_block(jj));
                mbar_arrive_expect_tx(&tl->v_full[st], kStageBytes);
                tma_load_3d(sv + st * kStageBytes, &tmap_v, &tl->v_full[st], 0, cr.x, cr.y);
                tma_load_3d(sv + st * kStageBytes + kBoxBytesKV, &tmap_v, &tl->v_full[st], 64, cr.x, cr.y);
                vk++;
            }
            for (int i = max(0, vk - kNV); i < vk; i++)  // copies in flight land before exit
                mbar_wait(&tl->v_full[i % kNV], (i / kNV) & 1, nullptr);
        }
    } else if (warp == 5) {
        // ------------------------------------------------------------- MMA issuer
        if (lane == 0 && nblk > 0) {
            constexpr uint32_t idesc_s = umma_idesc_bf16(128, kBN, 0);
            constexpr uint32_t idesc_pv = umma_idesc_bf16(128, 128, 1);
            constexpr uint32_t dhi = umma_desc_hi_sw128();
            const uint32_t q_lo = umma_desc_lo(smem_addr(sq), 16);
            const uint32_t k_lo = umma_desc_lo(smem_addr(sk), 16);
            const uint32_t v_lo = umma_desc_lo(smem_addr(sv), kBoxBytesKV);  // MN-major: LBO = box stride
            const uint32_t s_col = tmem, p_col = tmem + kColP, o_col = tmem + kColO;
            bool ok = mbar_wait(&tl->q_full, 0, &tl->abort);
            if (!ok) set_timeout(tl, p.status);
            auto issue_s = [&](int jj) {  // S = Q . K_jj^T, d = 128 in 8 steps of 16
                const uint32_t kst = k_lo + (uint32_t)(((jj % kNK) * kStageBytes) >> 4);
#pragma unroll
                for (int kk = 0; kk < 8; kk++) {
                    const uint32_t qo = (uint32_t)(((kk >> 2) * kBoxBytesQ + (kk & 3) * 32) >> 4);
                    const uint32_t ko = (uint32_t)(((kk >> 2) * kBoxBytesKV + (kk & 3) * 32) >> 4);
                    umma_ss2(s_col, q_lo + qo, kst + ko, dhi, idesc_s, kk > 0 ? 1u : 0u);
                }
                umma_commit(&tl->s_full);
                umma_commit(&tl->k_empty[jj % kNK]);  // K is read by S only
            };
            // S(ns) once the softmax holds S(ns-1) in registers and K(ns) landed; block
            // np's decision as it arrives (P.V when kept, then its V stage back)
            int n_pv = 0, ns = 0, np = 0, vk = 0;
            long long t_last = clock64();
            while (ok && np < nent) {
                bool did = false;
                if (ns < nent && (ns == 0 || mbar_test_wait(&tl->s_free, (ns - 1) & 1)) &&
                    mbar_test_wait(&tl->k_full[ns % kNK], (ns / kNK) & 1)) {
                    tc_fence_after();
                    issue_s(ns);
                    ns++;
                    did = true;
                }
                // (a kept block whose V has not landed yet waits here without holding up S)
                if (np < ns && mbar_test_wait(&tl->p_full[np % kDecRing], (np / kDecRing) & 1) &&
                    (CALIB || !dec[np] || mbar_test_wait(&tl->v_full[vk % kNV], (vk / kNV) & 1))) {
                    tc_fence_after();
                    if (!CALIB && dec[np]) {
                        const int st = vk % kNV;
                        const uint32_t vst = v_lo + (uint32_t)((st * kStageBytes) >> 4);
                        const uint32_t pb = p_col + (uint32_t)((n_pv & 1) * 32);
#pragma unroll
                        for (int kk = 0; kk < kBN / 16; kk++)
                            umma_ts2(o_col, pb + kk * 8, vst + (uint32_t)((kk * 16 * 128) >> 4), dhi, idesc_pv,
                                     (n_pv > 0 || kk > 0) ? 1u : 0u);
                        umma_commit(&tl->o_done[n_pv & 1]);
                        umma_commit(&tl->v_empty[st]);
                        n_pv++;
                        vk++;
                    }
                    mbar_arrive(&tl->dec_free[np % kDecRing]);
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
    } else if (warp < 4) {
        // ----------------------------------------------------- softmax / decision
        const int row = threadIdx.x;  // 0..127, TMEM lane
        const bool valid_row = row < p.R;
        const int pos = row % p.Lq;
        const int last_key = !valid_row ? -1 : (p.causal ? pos + Lk - p.Lq : Lk - 1);
        const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
        const uint32_t s_addr = tmem + lane_off, o_addr = tmem + lane_off + kColO;
        const float NEG_INF = -CUDART_INF_F;
        float m_true = NEG_INF, m_ref = NEG_INF, l = 0.f, lr = 0.f;
        int n_kept = 0;
        bool seen = seed != 0;  // a seeded split has no forced first block
        unsigned int n_skip = 0;
        uint32_t mword = 0;
        int mword_idx = -1;
        for (int jj = 0; jj < nent; jj++) {
            const int j = entry_block(jj);
            const int sl = jj % kDecRing;
            if (!mbar_wait(&tl->s_full, jj & 1, &tl->abort)) set_timeout(tl, p.status);
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
            // the MMA thread has taken the decision published kDecRing entries ago
            if (jj >= kDecRing && !mbar_wait(&tl->dec_free[sl], ((jj / kDecRing) - 1) & 1, &tl->abort))
                set_timeout(tl, p.status);
            if (seed && jj == 0) {
                // the seed block: its row maxima start the running max of this split
                m_true = mt;
                if (row == 0) {
                    dec[jj] = 0;
                    __threadfence_block();
                    *reinterpret_cast<volatile int *>(&tl->dec_count) = jj + 1;
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&tl->p_full[sl]);
                continue;
            }
            const float mn = fmaxf(m_true, mt);
            const bool vote = (mt == NEG_INF) || (mt - mn < p.thr_log2);
            const bool all = bar_and(1, 128, vote);
            // Every block of the split below the sequence's length is visited: row Lq-1 of
            // the first head sees keys up to Lk - 1 (bottom-right alignment).
            const bool visited = true;
            const bool first = visited && !seen;
            seen = seen || visited;
            const bool skip = visited && all && !first;
            const bool kept = visited && !skip;
            if (row == 0) {
                // the V producer reads the decision before this block's exponentials run
                dec[jj] = kept ? 1 : 0;
                __threadfence_block();
                *reinterpret_cast<volatile int *>(&tl->dec_count) = jj + 1;
            }
            if (CALIB && p.gaps) {
                float g = mt == NEG_INF ? NEG_INF : mt - mn;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) g = fmaxf(g, __shfl_xor_sync(0xffffffffu, g, o));
                if (lane == 0) tl->gred[warp] = g;
                bar_sync(1, 128);
                if (row == 0) {
                    const float gg = fmaxf(fmaxf(tl->gred[0], tl->gred[1]), fmaxf(tl->gred[2], tl->gred[3]));
                    p.gaps[(size_t)bh * p.nb + j] =
                        !visited ? CUDART_NAN_F : (first ? CUDART_INF_F : gg * 0.69314718055994531f);
                }
                bar_sync(1, 128);
            }
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
                // P buffer n_kept & 1 was last read by the P.V of kept block n_kept - 2;
                // rescaling O needs every earlier P.V done (they complete in issue order)
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
                    for (int c = 0; c < 4; c++) {
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
            if (row == 0 && p.skip_mask && skip) {
                if (mword_idx != (j >> 5)) {
                    if (mword_idx >= 0 && mword) atomicOr(p.skip_mask + (size_t)bh * p.words + mword_idx, mword);
                    mword_idx = j >> 5;
                    mword = 0;
                }
                mword |= 1u << (j & 31);
            }
        }
        if (row == 0) {
            if (p.skip_mask && mword_idx >= 0 && mword) atomicOr(p.skip_mask + (size_t)bh * p.words + mword_idx, mword);
            if (p.split_skips)
                p.split_skips[(size_t)bh * p.num_splits + split] = n_skip;
            else if (p.skip_count && n_skip)
                atomicAdd(p.skip_count, (unsigned long long)n_skip);
        }
        if (!CALIB) {
            // split epilogue: normalised partial O and the split's lse for each valid row
            const size_t orow = ((size_t)(b * p.Hq + hkv * p.G) * p.Lq + row) * p.num_splits + split;
            if (n_kept > 0) {
                if (!mbar_wait(&tl->o_done[(n_kept - 1) & 1], ((n_kept - 1) >> 1) & 1, &tl->abort))
                    set_timeout(tl, p.status);
                tc_fence_after();
            }
            const float inv = lr > 0.f ? 1.f / lr : 0.f;
#pragma unroll 1
            for (int c = 0; c < 4; c++) {
                uint32_t orr[32];
                if (nblk > 0) {
                    tmem_ld32(o_addr + c * 32, orr);
                    tc_wait_ld();
                }
                if (valid_row) {
                    float *dst = p.part_o + orow * 128 + c * 32;
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
            if (valid_row) p.part_lse[orow] = l > 0.f ? (m_ref + __log2f(l)) * 0.69314718055994531f : NEG_INF;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 5) tmem_dealloc(tmem, 256);
}

template <bool CALIB>
cudaError_t launch_t(const DecodeParams &p, const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                     cudaStream_t st) {
    constexpr int smem = wide_smem_bytes(CALIB);
    auto kern = decode_wide_kernel<CALIB>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    dim3 grid(p.num_splits, p.Hkv, p.B);
    kern<<<grid, kThreads, smem, st>>>(p, tq, tk, tv);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode_wide(const DecodeParams &p, const CUtensorMap &tq, const CUtensorMap &tk,
                               const CUtensorMap &tv, bool calib, cudaStream_t st) {
    return calib ? launch_t<true>(p, tq, tk, tv, st) : launch_t<false>(p, tq, tk, tv, st);
}

}  // namespace blasst
