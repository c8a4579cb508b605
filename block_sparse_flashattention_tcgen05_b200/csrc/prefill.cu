// prefill.cu -- tcgen05 prefill attention with softmax-threshold block skipping
// (BLASST), and the decision-only calibration pass that shares its pipeline.
//
// One CTA handles two 128-row query tiles (A, B) of one (sequence, query
// head) that share every K/V block it loads.  d = dv = 128, KV blocks of 128.
//
// Warp roles (352 threads):
//   warps 0-3  softmax/decision warpgroup for tile A (thread i owns row i,
//              i.e. TMEM lane i), warps 4-7 the same for tile B;
//   warp 8     TMA producer: Q_A and Q_B once, then K_j into a 3-stage ring;
//   warp 9     allocates TMEM and issues every tcgen05.mma from one thread;
//   warp 10    TMA producer for V_j (2-stage ring; V is loaded for every
//              block, as the prefill design of the pages keeps V prefetch
//              regular), separate so the K stream never waits on a V slot.
//
// TMEM (512 columns): S_A [0,128), S_B [128,256), O_A [256,384),
// O_B [384,512); P_t (bf16, 64 columns) overwrites the first half of S_t.
//
// Per tile and KV block j:
//   MMA:      S_t = Q_t K_j^T           (always, for every visited block)
//   softmax:  row max m~ of scale*S, true running max M <- max(M, m~),
//             vote (m~ - M < log2 lambda, or the row sees no key of the
//             block); the tile decision is the AND over the 128 rows, taken
//             in two levels: __all_sync per warp, then a named barrier that
//             only warps voting "skip" wait on (the others arrive and go on).
//             The first block is never skipped.
//   kept:     lazy rescale of O when the exp reference lags M by > 2^8,
//             P = 2^(s - M_ref) -> bf16 in TMEM, l += sum P, then
//             MMA: O_t += P_t V_j.
//   skipped:  no exp, no P, no P.V (xllm-io paper review, section 3
//             "prefill kernel optimisation": BMM1 always computed, exp and
//             BMM2 omitted for skipped blocks).
// The skip decision always uses the true running max; the exp reference
// M_ref may lag it (conditional rescaling), which changes nothing in exact
// arithmetic.
#include <cuda_bf16.h>
#include <math_constants.h>

#include "internal.h"
#include "ptx.cuh"

namespace blasst {
namespace {

constexpr int kThreads = 352;
constexpr int kSoftmaxThreads = 128;
constexpr int kProducerWarp = 8;   // Q and K
constexpr int kMmaWarp = 9;
constexpr int kVProducerWarp = 10;  // V
constexpr int kStagesK = 3;
constexpr int kStagesV = 2;
constexpr int kTileBytes = 128 * 128 * 2;  // 128 rows x 128 bf16
constexpr int kBoxBytes = kTileBytes / 2;  // 128 rows x 64 bf16 (one swizzle box)
constexpr float kRescaleThreshold = 8.0f;  // log2 units
constexpr int kStatusTimeout = 1;

struct PrefillSmemTail {
    uint64_t q_full;
    uint64_t k_full[kStagesK], k_empty[kStagesK];
    uint64_t v_full[kStagesV], v_empty[kStagesV];
    uint64_t s_full[2], p_full[2], o_done[2];
    uint64_t mma_done;
    uint32_t tmem_base;
    int dec[2];
    uint32_t votes[2][2];  // [tile][block parity]: byte w = warp w's rows all allow the skip
    int abort;
    float gred[2][4];
};

template <bool CALIB>
constexpr int prefill_smem_bytes() {
    return 2 * kTileBytes + kStagesK * kTileBytes + (CALIB ? 0 : kStagesV * kTileBytes) +
           (int)sizeof(PrefillSmemTail) + 1024;
}

__device__ __forceinline__ void set_timeout(PrefillSmemTail *t, unsigned int *status) {
    t->abort = 1;
    if (status) atomicOr(status, kStatusTimeout);
}

__device__ __forceinline__ int last_block(const PrefillParams &p, int q0) {
    if (q0 >= p.Lq) return -1;
    if (!p.causal) return p.nb - 1;
    const int last_row = min(p.Lq, q0 + 128) - 1;
    return min(p.nb - 1, (last_row + p.Lk - p.Lq) >> 7);
}

// MODE 0: attention; 1: decision-only calibration pass; 2: attention with the
// skip decision compiled out (every visited block kept, no vote, no barrier), a
// measurement instance that gives the cost of the decision at lambda = 0.
template <int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_kernel(const PrefillParams p, const __grid_constant__ CUtensorMap tmap_q,
                   const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v) {
    constexpr bool CALIB = MODE == 1;
    constexpr bool NOVOTE = MODE == 2;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sq = smem;                                  // Q_A, Q_B
    uint8_t *sk = smem + 2 * kTileBytes;                 // K ring
    uint8_t *sv = sk + kStagesK * kTileBytes;            // V ring
    PrefillSmemTail *tl = reinterpret_cast<PrefillSmemTail *>(sv + (CALIB ? 0 : kStagesV * kTileBytes));

    // longest rows first: blockIdx.x walks pairs of query tiles from the end
    const int n_pairs = (p.n_qtiles + 1) / 2;
    const int bhq = blockIdx.x % (p.B * p.Hq);
    const int pair = n_pairs - 1 - blockIdx.x / (p.B * p.Hq);
    const int b = bhq / p.Hq, hq = bhq % p.Hq;
    const int hkv = hq / p.G;
    const int q0[2] = {pair * 256, pair * 256 + 128};
    const int jmax[2] = {last_block(p, q0[0]), last_block(p, q0[1])};
    const int jmax_all = max(jmax[0], jmax[1]);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        mbar_init(&tl->q_full, 1);
        for (int i = 0; i < kStagesK; i++) {
            mbar_init(&tl->k_full[i], 1);
            mbar_init(&tl->k_empty[i], 1);
        }
        for (int i = 0; i < kStagesV; i++) {
            mbar_init(&tl->v_full[i], 1);
            mbar_init(&tl->v_empty[i], 1);
        }
        for (int t = 0; t < 2; t++) {
            mbar_init(&tl->s_full[t], 1);
            mbar_init(&tl->p_full[t], kSoftmaxThreads / 32);
            mbar_init(&tl->o_done[t], 1);
        }
        mbar_init(&tl->mma_done, 1);
        tl->abort = 0;
        fence_mbar_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(&tl->tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tl->tmem_base;

    if (warp == kProducerWarp) {
        // --------------------------------------------------------- TMA producer: Q, K
        if (lane == 0) {
            tma_prefetch_desc(&tmap_q);
            tma_prefetch_desc(&tmap_k);
            const int qrow = b * p.Hq + hq;
            const int nq = jmax[1] >= 0 ? 2 : 1;
            mbar_arrive_expect_tx(&tl->q_full, nq * kTileBytes);
            for (int t = 0; t < nq; t++) {
                tma_load_3d(sq + t * kTileBytes, &tmap_q, &tl->q_full, 0, q0[t], qrow);
                tma_load_3d(sq + t * kTileBytes + kBoxBytes, &tmap_q, &tl->q_full, 64, q0[t], qrow);
            }
            const int kvrow = b * p.Hkv + hkv;
            int issued = 0;
            for (int j = 0; j <= jmax_all && !tl->abort; j++) {
                const int st = j % kStagesK;
                if (j >= kStagesK && !mbar_wait(&tl->k_empty[st], ((j / kStagesK) & 1) ^ 1, &tl->abort)) {
                    set_timeout(tl, p.status);
                    break;
                }
                mbar_arrive_expect_tx(&tl->k_full[st], kTileBytes);
                tma_load_3d(sk + st * kTileBytes, &tmap_k, &tl->k_full[st], 0, j * 128, kvrow);
                tma_load_3d(sk + st * kTileBytes + kBoxBytes, &tmap_k, &tl->k_full[st], 64, j * 128, kvrow);
                issued++;
            }
            if (tl->abort) {  // let copies already issued land
                for (int j = max(0, issued - kStagesK); j < issued; j++)
                    mbar_wait(&tl->k_full[j % kStagesK], (j / kStagesK) & 1, nullptr);
            }
        }
    } else if (warp == kVProducerWarp) {
        // ------------------------------------------------------------ TMA producer: V
        if (!CALIB && lane == 0) {
            tma_prefetch_desc(&tmap_v);
            const int kvrow = b * p.Hkv + hkv;
            int issued = 0;
            for (int j = 0; j <= jmax_all && !tl->abort; j++) {
                const int st = j % kStagesV;
                // the stage is free once the MMA warp is done with its previous block and that
                // block's load has landed (a block every tile skipped is released unread)
                if (j >= kStagesV && (!mbar_wait(&tl->v_empty[st], ((j / kStagesV) & 1) ^ 1, &tl->abort) ||
                                      !mbar_wait(&tl->v_full[st], ((j / kStagesV) & 1) ^ 1, &tl->abort))) {
                    set_timeout(tl, p.status);
                    break;
                }
                mbar_arrive_expect_tx(&tl->v_full[st], kTileBytes);
                tma_load_3d(sv + st * kTileBytes, &tmap_v, &tl->v_full[st], 0, j * 128, kvrow);
                tma_load_3d(sv + st * kTileBytes + kBoxBytes, &tmap_v, &tl->v_full[st], 64, j * 128, kvrow);
                issued++;
            }
            // loads nobody waited for (blocks every tile skipped, or an abort) land before exit
            for (int j = max(0, issued - kStagesV); j < issued; j++)
                mbar_wait(&tl->v_full[j % kStagesV], (j / kStagesV) & 1, nullptr);
        }
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_s = umma_idesc_bf16(128, 128, 0);
            constexpr uint32_t idesc_pv = umma_idesc_bf16(128, 128, 1);
            int n_pv[2] = {0, 0};
            bool ok = mbar_wait(&tl->q_full, 0, &tl->abort);
            // descriptor low halves (start address | LBO); the high half is shared
            constexpr uint32_t dhi = umma_desc_hi_sw128();
            const uint32_t q_lo0 = umma_desc_lo(smem_addr(sq), 16);
            const uint32_t k_lo0 = umma_desc_lo(smem_addr(sk), 16);
            const uint32_t v_lo0 = umma_desc_lo(smem_addr(sv), kBoxBytes);
            auto issue_s = [&](int t, int j) {
                const uint32_t qa = q_lo0 + (uint32_t)t * (kTileBytes >> 4);
                const uint32_t ka = k_lo0 + (uint32_t)(j % kStagesK) * (kTileBytes >> 4);
                const uint32_t s_col = tmem + (uint32_t)t * 128u;
#pragma unroll
                for (int kk = 0; kk < 8; kk++) {
                    const uint32_t off = (uint32_t)((kk >> 2) * kBoxBytes + (kk & 3) * 32) >> 4;
                    umma_ss2(s_col, qa + off, ka + off, dhi, idesc_s, kk > 0);
                }
                umma_commit(&tl->s_full[t]);
            };
            // prologue: S_t(0)
            if (ok && jmax_all >= 0) {
                if (!mbar_wait(&tl->k_full[0], 0, &tl->abort)) ok = false;
                tc_fence_after();
                for (int t = 0; t < 2 && ok; t++)
                    if (jmax[t] >= 0) issue_s(t, 0);
                umma_commit(&tl->k_empty[0]);
            }
            for (int j = 0; j <= jmax_all && ok; j++) {
                const int st = j % kStagesV;
                bool v_waited = false;
                bool k_next_waited = false;
#pragma unroll
                for (int t = 0; t < 2; t++) {
                    if (j > jmax[t] || !ok) continue;
                    if (!mbar_wait(&tl->p_full[t], j & 1, &tl->abort)) {
                        set_timeout(tl, p.status);
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const bool kept = NOVOTE || (!CALIB && tl->dec[t] != 0);
                    if (kept) {
                        if (!v_waited) {
                            if (!mbar_wait(&tl->v_full[st], (j / kStagesV) & 1, &tl->abort)) {
                                set_timeout(tl, p.status);
                                ok = false;
                                break;
                            }
                            v_waited = true;
                        }
                        const uint32_t va = v_lo0 + (uint32_t)st * (kTileBytes >> 4);
                        const uint32_t s_col = tmem + (uint32_t)t * 128u;
                        const uint32_t o_col = tmem + 256u + (uint32_t)t * 128u;
                        const uint32_t acc0 = n_pv[t] > 0 ? 1u : 0u;
#pragma unroll
                        for (int kk = 0; kk < 8; kk++)
                            umma_ts2(o_col, s_col + kk * 8, va + kk * (2048 >> 4), dhi, idesc_pv,
                                     (acc0 || kk > 0) ? 1u : 0u);
                        umma_commit(&tl->o_done[t]);
                        n_pv[t]++;
                    }
                    if (j + 1 <= jmax[t]) {
                        if (!k_next_waited) {
                            if (!mbar_wait(&tl->k_full[(j + 1) % kStagesK], ((j + 1) / kStagesK) & 1, &tl->abort)) {
                                set_timeout(tl, p.status);
                                ok = false;
                                break;
                            }
                            k_next_waited = true;
                        }
                        // S_t(j+1) overwrites the columns that hold P_t(j).  tcgen05.mma
                        // operations issued by one thread execute in issue order, so the
                        // P.V above has read P before this product writes there.
                        issue_s(t, j + 1);
                    }
                }
                if (!ok) break;
                if (!CALIB) {
                    // V_j's stage goes back to the producer after the P.V that read it; when
                    // every tile skipped block j nothing here waits for its load (the producer
                    // does, before refilling the stage)
                    umma_commit(&tl->v_empty[st]);
                }
                if (k_next_waited) umma_commit(&tl->k_empty[(j + 1) % kStagesK]);
            }
            // every MMA and commit of this thread has completed before TMEM is released
            umma_commit(&tl->mma_done);
            if (!mbar_wait(&tl->mma_done, 0, nullptr)) set_timeout(tl, p.status);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------- softmax / decision
        const int t = warp >> 2;                 // tile of this warpgroup
        const int wq = warp & 3;                 // TMEM lane quadrant
        const int row = threadIdx.x & 127;       // tile row == TMEM lane
        const int bar_id = 1 + t;
        const int q0t = pair * 256 + t * 128;
        const int jmaxt = last_block(p, q0t);
        const int qpos = q0t + row;
        const bool valid_row = qpos < p.Lq;
        const int last_key = !valid_row ? -1 : (p.causal ? qpos + p.Lk - p.Lq : p.Lk - 1);
        const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
        const uint32_t s_addr = tmem + lane_off + (t ? 128u : 0u);
        const uint32_t o_addr = tmem + lane_off + (t ? 384u : 256u);
        const float NEG_INF = -CUDART_INF_F;
        const size_t tile_idx = ((size_t)b * p.Hq + hq) * p.n_qtiles + (q0t >> 7);
        // l: exact fp32 row sum (for lse); lr: sum of the bf16-rounded P that P.V
        // uses (normalises O, so a dominant key reproduces its value exactly)
        float m_true = NEG_INF, m_ref = NEG_INF, l = 0.f, lr = 0.f;
        int n_kept = 0;
        uint32_t mword = 0;
        unsigned int n_skip = 0;

        for (int j = 0; j <= jmaxt; j++) {
            if (!mbar_wait(&tl->s_full[t], j & 1, &tl->abort)) set_timeout(tl, p.status);
            tc_fence_after();
            uint32_t sr[128];
#pragma unroll
            for (int c = 0; c < 4; c++) tmem_ld32(s_addr + c * 32, sr + c * 32);
            tc_wait_ld();
            float *s = reinterpret_cast<float *>(sr);
            const int lim = last_key - j * 128;  // keys c <= lim are visible to this row
            if (lim < 127) {
#pragma unroll
                for (int c = 0; c < 128; c++)
                    if (c > lim) s[c] = NEG_INF;
            }
            // row max: four independent chains of 3-input max
            float m0 = NEG_INF, m1 = NEG_INF, m2 = NEG_INF, m3 = NEG_INF;
#pragma unroll
            for (int c = 0; c < 128; c += 8) {
                m0 = fmax3(m0, s[c], s[c + 1]);
                m1 = fmax3(m1, s[c + 2], s[c + 3]);
                m2 = fmax3(m2, s[c + 4], s[c + 5]);
                m3 = fmax3(m3, s[c + 6], s[c + 7]);
            }
            const float mx = fmax3(m0, m1, fmaxf(m2, m3));
            const float mt = mx * p.scale_log2;  // -inf stays -inf (scale > 0)
            const float mn = fmaxf(m_true, mt);
            const bool vote = (mt == NEG_INF) || (mt - mn < p.thr_log2);
            // Tile-wide AND in two levels.  A warp with a row that forbids the skip
            // knows the block is kept: it leaves its vote and arrives at the tile's named
            // barrier without waiting.  Only warps whose rows all allow the skip wait
            // there for the other three votes.  The first block is always kept and takes
            // no vote.  (A warp reaches block j+1 only after all four warps published block
            // j, so a barrier instance is complete before its id is used again; the ids
            // also alternate with the block parity.)
            bool skip = false;
            if (!NOVOTE && j > 0) {
                const bool wvote = __all_sync(0xffffffffu, vote);
                uint8_t *vb = reinterpret_cast<uint8_t *>(&tl->votes[t][j & 1]);
                if (lane == 0) vb[wq] = wvote ? 1 : 0;
                const int vid = 3 + 2 * t + (j & 1);
                if (wvote) {
                    bar_sync(vid, kSoftmaxThreads);
                    skip = *reinterpret_cast<volatile uint32_t *>(vb) == 0x01010101u;
                } else {
                    bar_arrive(vid, kSoftmaxThreads);
                }
            }
            if (CALIB && p.gaps) {
                float g = mt == NEG_INF ? NEG_INF : mt - mn;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) g = fmaxf(g, __shfl_xor_sync(0xffffffffu, g, o));
                if (lane == 0) tl->gred[t][wq] = g;
                bar_sync(bar_id, kSoftmaxThreads);
                if (row == 0) {
                    const float gg = fmaxf(fmaxf(tl->gred[t][0], tl->gred[t][1]), fmaxf(tl->gred[t][2], tl->gred[t][3]));
                    p.gaps[tile_idx * p.nb + j] = j == 0 ? CUDART_INF_F : gg * 0.69314718055994531f;
                }
                bar_sync(bar_id, kSoftmaxThreads);
            }
            if (!NOVOTE && row == 0) tl->dec[t] = skip ? 0 : 1;
            if (skip || CALIB) {
                if (!skip) m_true = mn;
                __syncwarp();
                if (lane == 0) mbar_arrive(&tl->p_full[t]);
                if (skip) {
                    n_skip++;
                    mword |= 1u << (j & 31);
                }
                if (row == 0 && p.skip_mask && ((j & 31) == 31 || j == jmaxt))
                    p.skip_mask[tile_idx * p.words + (j >> 5)] = mword;
                if ((j & 31) == 31) mword = 0;
                continue;
            }
            if (row == 0 && p.skip_mask && ((j & 31) == 31 || j == jmaxt))
                p.skip_mask[tile_idx * p.words + (j >> 5)] = mword;
            if ((j & 31) == 31) mword = 0;
            m_true = mn;
            // conditional rescale: only when the exp reference lags the true max by > 2^8
            const bool need = mn - m_ref > kRescaleThreshold;
            const bool warp_need = __any_sync(0xffffffffu, need);
            float alpha = 1.f;
            if (warp_need) {
                const float m_new = mn;
                alpha = (m_ref == NEG_INF || m_new == NEG_INF) ? (m_new == NEG_INF ? 1.f : 0.f) : ex2(m_ref - m_new);
                l *= alpha;
                lr *= alpha;
                if (m_new != NEG_INF) m_ref = m_new;
            }
            const float mref = m_ref == NEG_INF ? 0.f : m_ref;
            const uint64_t scl2 = f2_pack(p.scale_log2, p.scale_log2);
            const uint64_t neg2 = f2_pack(-mref, -mref);
            uint64_t rs2a = 0, rs2b = 0, rr2a = 0, rr2b = 0;  // packed {lo, hi} partial sums (0 == +0.0f pair)
#pragma unroll
            for (int h = 0; h < 4; h++) {  // P in four chunks of 32 keys (16 packed columns)
                uint32_t pk[16];
#pragma unroll
                for (int c = 0; c < 16; c++) {
                    const uint64_t y = f2_fma(f2_pack(s[h * 32 + 2 * c], s[h * 32 + 2 * c + 1]), scl2, neg2);
                    float y0, y1;
                    f2_unpack(y, y0, y1);
                    const float p0 = ex2(y0), p1 = ex2(y1);
                    pk[c] = pack_bf16x2(p0, p1);
                    if (c & 1) {
                        rs2b = f2_add(rs2b, f2_pack(p0, p1));
                        rr2b = f2_add(rr2b, bf16x2_widen(pk[c]));
                    } else {
                        rs2a = f2_add(rs2a, f2_pack(p0, p1));
                        rr2a = f2_add(rr2a, bf16x2_widen(pk[c]));
                    }
                }
                tmem_st16(s_addr + h * 16, pk);
            }
            {
                float a0, a1, b0, b1;
                f2_unpack(f2_add(rs2a, rs2b), a0, a1);
                f2_unpack(f2_add(rr2a, rr2b), b0, b1);
                l += a0 + a1;
                lr += b0 + b1;
            }
            // O rescale after P is out of registers; P.V(j) is issued only after p_full
            if (warp_need && n_kept > 0) {
                if (!mbar_wait(&tl->o_done[t], (n_kept - 1) & 1, &tl->abort)) set_timeout(tl, p.status);
                tc_fence_after();
#pragma unroll
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
            if (lane == 0) mbar_arrive(&tl->p_full[t]);
            n_kept++;
        }
        if (jmaxt >= 0) {
            if (row == 0 && p.skip_mask) {
                for (int w = (jmaxt >> 5) + 1; w < p.words; w++) p.skip_mask[tile_idx * p.words + w] = 0u;
            }
            if (CALIB && row == 0 && p.gaps) {
                for (int j = jmaxt + 1; j < p.nb; j++) p.gaps[tile_idx * p.nb + j] = CUDART_NAN_F;
            }
            if (row == 0 && p.skip_count && n_skip) atomicAdd(p.skip_count, (unsigned long long)n_skip);
        }
        if (!CALIB && jmaxt >= 0) {
            // epilogue: O / l -> bf16, lse = (M_ref + log2 l) * ln 2
            if (!mbar_wait(&tl->o_done[t], (n_kept - 1) & 1, &tl->abort)) set_timeout(tl, p.status);
            tc_fence_after();
            const float inv = lr > 0.f ? 1.f / lr : 0.f;
            uint16_t *orow = p.o + (((size_t)b * p.Hq + hq) * p.Lq + (valid_row ? qpos : 0)) * 128;
#pragma unroll
            for (int c = 0; c < 4; c++) {
                uint32_t orr[32];
                tmem_ld32(o_addr + c * 32, orr);
                tc_wait_ld();
                if (valid_row) {
#pragma unroll
                    for (int i = 0; i < 32; i += 8) {
                        uint4 v;
                        v.x = pack_bf16x2(__uint_as_float(orr[i + 0]) * inv, __uint_as_float(orr[i + 1]) * inv);
                        v.y = pack_bf16x2(__uint_as_float(orr[i + 2]) * inv, __uint_as_float(orr[i + 3]) * inv);
                        v.z = pack_bf16x2(__uint_as_float(orr[i + 4]) * inv, __uint_as_float(orr[i + 5]) * inv);
                        v.w = pack_bf16x2(__uint_as_float(orr[i + 6]) * inv, __uint_as_float(orr[i + 7]) * inv);
                        *reinterpret_cast<uint4 *>(orow + c * 32 + i) = v;
                    }
                }
            }
            if (valid_row)
                p.lse[((size_t)b * p.Hq + hq) * p.Lq + qpos] =
                    l > 0.f ? (m_ref + __log2f(l)) * 0.69314718055994531f : NEG_INF;
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kMmaWarp) tmem_dealloc(tmem, 512);
}

template <int MODE>
cudaError_t launch_t(const PrefillParams &p, const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                     cudaStream_t st) {
    constexpr int smem = prefill_smem_bytes<MODE == 1>();
    auto kern = prefill_kernel<MODE>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    const int n_pairs = (p.n_qtiles + 1) / 2;
    dim3 grid(n_pairs * p.B * p.Hq);
    kern<<<grid, kThreads, smem, st>>>(p, tq, tk, tv);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill(const PrefillParams &p, const CUtensorMap &tq, const CUtensorMap &tk,
                           const CUtensorMap &tv, bool calib, cudaStream_t st) {
    return calib ? launch_t<1>(p, tq, tk, tv, st) : launch_t<0>(p, tq, tk, tv, st);
}

cudaError_t launch_prefill_novote(const PrefillParams &p, const CUtensorMap &tq, const CUtensorMap &tk,
                                  const CUtensorMap &tv, cudaStream_t st) {
    return launch_t<2>(p, tq, tk, tv, st);
}

}  // namespace blasst
