// backward.cu -- attention backward for the prefill tiling with the forward's
// skip mask held fixed: skipped (query tile, KV block) pairs get no gradient,
// which is the optional sparsity-aware training of the pages (xllm-io paper
// review, section 3, "training procedure": the forward skips blocks, the
// skipped blocks receive no gradient in the backward pass).
//
// Three launches:
//   prep      per query row: -scale * rowsum(dO * O) and -lse*log2(e) (fp32;
//             -inf on padding rows and rows that saw no key, so their P is 0),
//             and the row of the fp32 dQ accumulator set to zero;
//   main      one CTA per (KV block j of 128 keys, KV head, sequence) walks the
//             kept (query tile i, query head) pairs of its KV head in order
//             and accumulates dK_j and dV_j over all of them in tensor memory;
//             dQ_i contributions go to the fp32 accumulator by bulk reduce-add
//             (cp.reduce.async.bulk .add.f32, two 32 KB row ranges per pair)
//             from shared memory, staged by the compute warps in the pair's
//             Q and dO stages;
//   finalize  dQ accumulator -> bf16 dq.
//
// Main kernel, per pair (S^T etc. are key-major: TMEM lane = key of block j):
//   S^T  = K_j Q_i^T                        tcgen05, A = K (K-major), B = Q (K-major)
//   dP^T = V_j dO_i^T                       tcgen05, A = V, B = dO (both K-major)
//   P^T  = 2^(S^T * scale*log2e - lse*log2e)  masked (key >= Lk, causal) to 0
//   dS^T = P^T (scale*dP^T - scale*D)       bf16 into shared memory
//   dQ^T = K_j^T dS^T                       A = K (MN-major), B = dS^T (MN-major)
//   dV  += P^T dO_i                         A = P^T from TMEM (bf16), B = dO (MN-major)
//   dK  += dS^T Q_i                         A = dS^T (K-major), B = Q (MN-major)
//
// Warp roles:
//   compute    4 * kColGroups warps: warp w owns TMEM lanes 32*(w%4).. (keys
//              for S^T/dP^T, head dims for dQ^T) and column group w/4 (128 /
//              kColGroups columns);
//   producer   TMA: K_j, V_j once; Q_i, dO_i and the two per-row vectors per
//              pair into a 2-stage ring;
//   MMA        allocates TMEM and issues every tcgen05.mma from one thread;
//   reduce     issues the bulk reduce-add of each pair's staged dQ rows.
//
// TMEM (512 columns): S^T [0,128) -> P^T (bf16; each column group's P^T packed
// into the first half of its own S^T columns); dP^T [128,256) -> dQ^T;
// dV [256,384); dK [384,512).
//
// MMA issue order per pair t: dP(t) [after the dQ^T(t-1) columns are read],
// then, once dS^T(t) is ready: dQ^T(t), dK(t), dV(t), S(t+1).  Operations
// issued by one thread execute in issue order, so S(t+1) overwrites P^T(t) only
// after dV(t) has read it, and a commit covers every earlier operation.
// dQ staging: pair t's Q stage is not read again once dK(t) has completed, nor
// its dO stage once dV(t) has, and they take dQ(t) as fp32 rows (queries 0-63
// in the Q stage while the tensor core runs dV(t), 64-127 in the dO stage while
// it runs S(t+1); 512 bytes of head dims per row, the accumulator's own layout).  The reduce
// warp adds both ranges to the accumulator and hands the stages back to the
// producer for pair t+2 (stage_free) once the bulk copies have read them.
// Nothing on the compute warps' path waits for the reduction (staging in the
// dS^T buffer instead, whose reuse for dS(t+1) then waited on it, measured
// 8 % slower dense).
#include <climits>

#include <cuda_bf16.h>
#include <math_constants.h>

#include "internal.h"
#include "ptx.cuh"

namespace blasst {
namespace {

#ifndef BLASST_BWD_COL_GROUPS
#define BLASST_BWD_COL_GROUPS 4
#endif
// The 128 columns of a pair are split into kColGroups groups; a compute warp owns
// one TMEM lane quadrant and one group, so there are 4 * kColGroups compute warps.
constexpr int kColGroups = BLASST_BWD_COL_GROUPS;
constexpr int kCW = 128 / kColGroups;  // columns per compute warp (64 or 32)
constexpr int kChunks = kCW / 32;      // 32-column TMEM loads per operand
constexpr int kComputeWarps = 4 * kColGroups;
constexpr int kProducerWarp = kComputeWarps;
constexpr int kMmaWarp = kComputeWarps + 1;
constexpr int kReduceWarp = kComputeWarps + 2;
constexpr int kThreads = 32 * (kComputeWarps + 3);
static_assert(kColGroups == 2 || kColGroups == 4, "64 or 32 columns per compute warp");
constexpr int kTileBytes = 128 * 128 * 2;  // 128 rows x 128 bf16
constexpr int kBoxBytes = kTileBytes / 2;  // 128 rows x 64 bf16 (one 128-byte swizzle box)
constexpr int kStatusTimeout = 1;
constexpr int kStatusSmemAlign = 4;
// CTA order for long sequences (at least kOrderMinBlocks KV blocks): chunks of kOrderChunk
// consecutive KV blocks, one KV head after another within a chunk, chunks in block order.
// Blocks with more query tiles (causal: small j) still start early, and the CTAs resident
// together mostly share one or two KV heads, so their Q, dO tiles and dQ accumulator rows
// are reused in L2 (32K causal GQA: DRAM traffic per launch 19.8 -> 8.1 GB dense and
// 30.6 -> 22.7 GB at 75 %).  Shorter sequences keep the KV head as the fastest index: there
// a chunk is a large share of the blocks, and the longest CTAs of the last heads would
// start too late (16K: 16 % slower with chunks of 64).
constexpr int kOrderChunk = 64;
constexpr int kOrderMinBlocks = 256;

struct BwdTail {
    float nl2[2][128];  // per stage: -lse * log2(e) of the pair's 128 query rows
    float nsd[2][128];  // per stage: -scale * rowsum(dO * O)
    uint64_t kv_full;
    uint64_t qdo_full[2], qdo_empty[2];
    uint64_t s_full, dp_full, ds_ready, dq_full, dq_free, acc_done;
    // [stage]: the compute warps have written dQ(t)'s rows to pair t's Q and dO stages.  One
    // barrier per stage: the compute warps may stage pair t+1 before the reduce warp has seen
    // pair t's phase, but pair t+2 (the same stage) only after the stage came back (stage_free).
    uint64_t dq_staged[2];
    uint64_t stage_free[2];  // [stage]: the bulk reduce of dQ(t) has read the staged rows
    uint64_t dk_done;        // dK(t) has completed: pair t's Q stage takes dQ(t)'s rows 0-63
    uint32_t tmem_base;
    int abort;
};

// K_j, V_j, Q/dO stages, dS^T; the base is 1024-byte aligned (checked)
constexpr int kSmemBytes = 7 * kTileBytes + (int)sizeof(BwdTail);

__device__ __forceinline__ void set_timeout(BwdTail *t, unsigned int *status) {
    t->abort = 1;
    if (status) atomicOr(status, kStatusTimeout);
}

// First query tile whose rows see a key of block j (tiles before it are not
// visited by the forward for this block).
__device__ __forceinline__ int first_tile(const BwdParams &p, int j) {
    if (!p.causal) return 0;
    const int need = j * 128 - (p.Lk - p.Lq) - 127;  // tile i qualifies iff i*128 >= need
    return need <= 0 ? 0 : (need + 127) / 128;
}

// From (i, g) inclusive, move to the next pair (tile i, head g of the group)
// that the forward kept for block j.  False when none is left.
__device__ __forceinline__ bool next_pair(const BwdParams &p, int b, int hkv, int j, int &i, int &g) {
    while (i < p.nq) {
        if (!p.skip_mask) return true;
        const int hq = hkv * p.G + g;
        const uint32_t w = __ldg(p.skip_mask + (((size_t)b * p.Hq + hq) * p.nq + i) * p.words + (j >> 5));
        if (!((w >> (j & 31)) & 1u)) return true;
        if (++g == p.G) {
            g = 0;
            ++i;
        }
    }
    return false;
}

// Bounded wait whose outcome is the same on every lane of the warp: the compute
// warps issue warp-collective TMEM loads and stores after their waits, so a lane
// must never leave a loop that the rest of its warp stays in.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, volatile int *abort) {
    return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort));
}

__device__ __forceinline__ void advance(const BwdParams &p, int &i, int &g) {
    if (++g == p.G) {
        g = 0;
        ++i;
    }
}

__global__ void __launch_bounds__(kThreads, 1)
    bwd_kernel(const BwdParams p, const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_do,
               const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v) {
    extern __shared__ __align__(1024) uint8_t smem[];
    if (smem_addr(smem) & 1023u) {  // the swizzled tiles need a 1024-byte aligned base
        if (threadIdx.x == 0 && p.status) atomicOr(p.status, kStatusSmemAlign);
        return;
    }
    uint8_t *sK = smem;
    uint8_t *sV = smem + kTileBytes;
    uint8_t *sQ = smem + 2 * kTileBytes;   // 2 stages
    uint8_t *sdO = smem + 4 * kTileBytes;  // 2 stages
    uint8_t *sdS = smem + 6 * kTileBytes;  // dS^T: [128 keys][128 queries] as two 64-query boxes
    BwdTail *tl = reinterpret_cast<BwdTail *>(smem + 7 * kTileBytes);

    int j, hkv;
    {
        const int chunk = p.nb >= kOrderMinBlocks ? kOrderChunk : 1;
        const int q = blockIdx.x / (chunk * p.Hkv), r = blockIdx.x % (chunk * p.Hkv);
        const int cq = min(chunk, p.nb - q * chunk);  // blocks in this chunk
        hkv = r / cq;
        j = q * chunk + r % cq;
    }
    const int b = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int kvrow = b * p.Hkv + hkv;

    if (threadIdx.x == 0) {
        mbar_init(&tl->kv_full, 1);
        for (int s = 0; s < 2; s++) {
            mbar_init(&tl->qdo_full[s], 1);
            mbar_init(&tl->qdo_empty[s], 1);
        }
        mbar_init(&tl->s_full, 1);
        mbar_init(&tl->dp_full, 1);
        mbar_init(&tl->ds_ready, kComputeWarps);
        mbar_init(&tl->dq_full, 1);
        mbar_init(&tl->dq_free, kComputeWarps);
        mbar_init(&tl->acc_done, 1);
        mbar_init(&tl->dk_done, 1);
        mbar_init(&tl->dq_staged[0], kComputeWarps);
        mbar_init(&tl->dq_staged[1], kComputeWarps);
        mbar_init(&tl->stage_free[0], 1);
        mbar_init(&tl->stage_free[1], 1);
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
    int n_steps = 0;  // pairs processed (compute warps: for the epilogue)

    if (warp == kProducerWarp) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            tma_prefetch_desc(&tmap_q);
            tma_prefetch_desc(&tmap_do);
            tma_prefetch_desc(&tmap_k);
            tma_prefetch_desc(&tmap_v);
            mbar_arrive_expect_tx(&tl->kv_full, 2 * kTileBytes);
            tma_load_3d(sK, &tmap_k, &tl->kv_full, 0, j * 128, kvrow);
            tma_load_3d(sK + kBoxBytes, &tmap_k, &tl->kv_full, 64, j * 128, kvrow);
            tma_load_3d(sV, &tmap_v, &tl->kv_full, 0, j * 128, kvrow);
            tma_load_3d(sV + kBoxBytes, &tmap_v, &tl->kv_full, 64, j * 128, kvrow);
            int i = first_tile(p, j), g = 0, t = 0;
            while (!tl->abort && next_pair(p, b, hkv, j, i, g)) {
                const int st = t & 1;
                // the stage held pair t-2: the tensor core is done with it and the dQ rows staged
                // in its Q tile have been read by the bulk reduce
                if (t >= 2 && (!mbar_wait(&tl->qdo_empty[st], ((t >> 1) & 1) ^ 1, &tl->abort) ||
                               !mbar_wait(&tl->stage_free[st], ((t >> 1) & 1) ^ 1, &tl->abort))) {
                    set_timeout(tl, p.status);
                    break;
                }
                const int qrow = b * p.Hq + hkv * p.G + g;
                const size_t rbase = (size_t)qrow * p.Lq_pad + (size_t)i * 128;
                mbar_arrive_expect_tx(&tl->qdo_full[st], 2 * kTileBytes + 2 * 512);
                uint8_t *q_dst = sQ + st * kTileBytes;
                uint8_t *do_dst = sdO + st * kTileBytes;
                tma_load_3d(q_dst, &tmap_q, &tl->qdo_full[st], 0, i * 128, qrow);
                tma_load_3d(q_dst + kBoxBytes, &tmap_q, &tl->qdo_full[st], 64, i * 128, qrow);
                tma_load_3d(do_dst, &tmap_do, &tl->qdo_full[st], 0, i * 128, qrow);
                tma_load_3d(do_dst + kBoxBytes, &tmap_do, &tl->qdo_full[st], 64, i * 128, qrow);
                bulk_load(&tl->nl2[st][0], p.neg_lse2 + rbase, 512, &tl->qdo_full[st]);
                bulk_load(&tl->nsd[st][0], p.neg_sdelta + rbase, 512, &tl->qdo_full[st]);
                t++;
                advance(p, i, g);
            }
            // loads nobody will wait for (after an abort) land before the CTA exits
            mbar_wait(&tl->kv_full, 0, nullptr);
            if (tl->abort)
                for (int u = max(0, t - 2); u < t; u++) mbar_wait(&tl->qdo_full[u & 1], (u >> 1) & 1, nullptr);
        }
        __syncwarp();
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t dhi = umma_desc_hi_sw128();
            constexpr uint32_t idesc_kk = umma_idesc_bf16_mn(128, 128, 0, 0);  // S^T, dP^T
            constexpr uint32_t idesc_kmn = umma_idesc_bf16_mn(128, 128, 0, 1); // dV (A in TMEM), dK
            constexpr uint32_t idesc_mnmn = umma_idesc_bf16_mn(128, 128, 1, 1);  // dQ^T
            // K-major operands: 16-wide K steps inside a 64-wide swizzle box, then the next box
            const uint32_t k_km = umma_desc_lo(smem_addr(sK), 16);
            const uint32_t v_km = umma_desc_lo(smem_addr(sV), 16);
            const uint32_t q_km = umma_desc_lo(smem_addr(sQ), 16);
            const uint32_t do_km = umma_desc_lo(smem_addr(sdO), 16);
            const uint32_t ds_km = umma_desc_lo(smem_addr(sdS), 16);
            // MN-major operands: the two 64-wide MN boxes are kBoxBytes apart; a K step is 16 rows
            const uint32_t k_mn = umma_desc_lo(smem_addr(sK), kBoxBytes);
            const uint32_t q_mn = umma_desc_lo(smem_addr(sQ), kBoxBytes);
            const uint32_t do_mn = umma_desc_lo(smem_addr(sdO), kBoxBytes);
            const uint32_t ds_mn = umma_desc_lo(smem_addr(sdS), kBoxBytes);
            constexpr uint32_t kStage16 = kTileBytes >> 4;
            auto koff = [](int kk) { return (uint32_t)((kk >> 2) * kBoxBytes + (kk & 3) * 32) >> 4; };
            auto issue_s = [&](int st) {  // S^T = K Q^T into [0,128)
#pragma unroll
                for (int kk = 0; kk < 8; kk++)
                    umma_ss2(tmem, k_km + koff(kk), q_km + st * kStage16 + koff(kk), dhi, idesc_kk, kk > 0);
            };
            bool ok = mbar_wait(&tl->kv_full, 0, &tl->abort);
            int i = first_tile(p, j), g = 0, t = 0;
            bool have = ok && next_pair(p, b, hkv, j, i, g);
            if (have) {
                if (!mbar_wait(&tl->qdo_full[0], 0, &tl->abort)) {
                    set_timeout(tl, p.status);
                    have = false;
                } else {
                    tc_fence_after();
                    issue_s(0);
                    umma_commit(&tl->s_full);
                }
            }
            while (have) {
                const int st = t & 1;
                // dP^T(t) = V dO^T into [128,256), once dQ^T(t-1) has been read out
                if (t > 0 && !mbar_wait(&tl->dq_free, (t - 1) & 1, &tl->abort)) {
                    set_timeout(tl, p.status);
                    break;
                }
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; kk++)
                    umma_ss2(tmem + 128, v_km + koff(kk), do_km + st * kStage16 + koff(kk), dhi, idesc_kk, kk > 0);
                umma_commit(&tl->dp_full);
                // the next pair (a mask lookup in global memory) while dS^T(t) is formed
                int ni = i, ng = g;
                advance(p, ni, ng);
                const bool more = next_pair(p, b, hkv, j, ni, ng);
                const int nst = (t + 1) & 1;
                if (!mbar_wait(&tl->ds_ready, t & 1, &tl->abort)) {
                    set_timeout(tl, p.status);
                    break;
                }
                tc_fence_after();
                // dQ^T = K^T dS^T (K = 128 keys) into [128,256)
#pragma unroll
                for (int kk = 0; kk < 8; kk++)
                    umma_ss2(tmem + 128, k_mn + kk * (2048 >> 4), ds_mn + kk * (2048 >> 4), dhi, idesc_mnmn, kk > 0);
                umma_commit(&tl->dq_full);
                // dK += dS^T Q (K = 128 queries)
#pragma unroll
                for (int kk = 0; kk < 8; kk++)
                    umma_ss2(tmem + 384, ds_km + koff(kk), q_mn + st * kStage16 + kk * (2048 >> 4), dhi, idesc_kmn,
                             (t > 0 || kk > 0) ? 1u : 0u);
                umma_commit(&tl->dk_done);  // pair t's Q stage: free for dQ(t)'s rows 0-63
                // dV += P^T dO (K = 128 queries; P^T of each column group in its own S^T columns)
#pragma unroll
                for (int kk = 0; kk < 8; kk++)
                    umma_ts2(tmem + 256, tmem + (uint32_t)((kk * 16 / kCW) * kCW + (kk * 16 % kCW) / 2),
                             do_mn + st * kStage16 + kk * (2048 >> 4), dhi, idesc_kmn, (t > 0 || kk > 0) ? 1u : 0u);
                umma_commit(&tl->qdo_empty[st]);  // pair t's Q and dO stages: free for dQ(t)'s rows
                // the next pair's S^T (overwrites P^T(t), which dV(t) above has read)
                if (more) {
                    if (!mbar_wait(&tl->qdo_full[nst], ((t + 1) >> 1) & 1, &tl->abort)) {
                        set_timeout(tl, p.status);
                        break;
                    }
                    tc_fence_after();
                    issue_s(nst);
                    umma_commit(&tl->s_full);
                }
                t++;
                i = ni;
                g = ng;
                have = more;
            }
            // every MMA of this thread has completed: dK, dV final, TMEM free to release
            umma_commit(&tl->acc_done);
        }
        __syncwarp();
    } else if (warp == kReduceWarp) {
        // ----------------------------------------------------------- dQ bulk reduce
        if (lane == 0) {
            int i = first_tile(p, j), g = 0, t = 0;
            while (!tl->abort && next_pair(p, b, hkv, j, i, g)) {
                const int st = t & 1;
                if (!mbar_wait(&tl->dq_staged[st], (t >> 1) & 1, &tl->abort)) {
                    set_timeout(tl, p.status);
                    break;
                }
                const int qrow = b * p.Hq + hkv * p.G + g;
                float *dst = p.dq_acc + ((size_t)qrow * p.Lq_pad + (size_t)i * 128) * 128;
                bulk_reduce_add_f32(dst, sQ + st * kTileBytes, 64 * 128 * 4);
                bulk_reduce_add_f32(dst + 64 * 128, sdO + st * kTileBytes, 64 * 128 * 4);
                bulk_commit_group();
                bulk_wait_read_all();
                mbar_arrive(&tl->stage_free[st]);
                t++;
                advance(p, i, g);
            }
            bulk_wait_all();  // every addition has been performed before the CTA exits
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ compute warps
        const int wq = warp & 3;   // TMEM lane quadrant
        const int hh = warp >> 2;  // column group: columns kCW*hh .. kCW*hh + kCW - 1
        const int r = wq * 32 + lane;  // TMEM lane: key row of the block (S^T, dP^T), head dim (dQ^T)
        const int key = j * 128 + r;
        const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
        const int shift = p.Lk - p.Lq;
        int i = first_tile(p, j), g = 0, t = 0;
        while (__all_sync(0xffffffffu, !tl->abort && next_pair(p, b, hkv, j, i, g))) {
            const int st = t & 1;
            const int q0 = i * 128 + hh * kCW;  // first query row of my columns
            if (!warp_wait(&tl->qdo_full[st], (t >> 1) & 1, &tl->abort) ||
                !warp_wait(&tl->s_full, t & 1, &tl->abort)) {
                set_timeout(tl, p.status);
                break;
            }
            tc_fence_after();
            const float *nl2 = &tl->nl2[st][hh * kCW];
            const float *nsd = &tl->nsd[st][hh * kCW];
            // Masking is needed only where some key of the block is past Lk or, causal,
            // past the first query of my columns (key <= q + shift); warp-uniform.
            const bool masked = (j * 128 + 128 > p.Lk) || (p.causal && j * 128 + 127 > q0 + shift);
            const int qmin = p.causal ? key - shift : INT_MIN;  // visible iff q >= qmin
            const bool key_ok = key < p.Lk;
            const uint64_t c2 = f2_pack(p.scale_log2, p.scale_log2);
            uint64_t pf[kCW / 2];  // P of my columns, as packed pairs
#pragma unroll
            for (int c = 0; c < kChunks; c++) {
                uint32_t sr[32];
                tmem_ld32(tmem + lane_off + (uint32_t)(hh * kCW + c * 32), sr);
                tc_wait_ld();
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 32; e += 2) {
                    const int cc = c * 32 + e;
                    float x0, x1;
                    f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[e]), __uint_as_float(sr[e + 1])), c2,
                                     *reinterpret_cast<const uint64_t *>(nl2 + cc)),
                              x0, x1);
                    if (masked) {
                        if (!(key_ok && q0 + cc >= qmin)) x0 = -CUDART_INF_F;
                        if (!(key_ok && q0 + cc + 1 >= qmin)) x1 = -CUDART_INF_F;
                    }
                    const float p0 = ex2(x0), p1 = ex2(x1);
                    pf[cc >> 1] = f2_pack(p0, p1);
                    pk[e >> 1] = pack_bf16x2(p0, p1);
                }
                // P^T (bf16) over columns this thread has already read
                tmem_st16(tmem + lane_off + (uint32_t)(hh * kCW + c * 16), pk);
            }
            if (!warp_wait(&tl->dp_full, t & 1, &tl->abort)) {
                set_timeout(tl, p.status);
                break;
            }
            tc_fence_after();
            // dS^T row r, my queries -> their 64-query box of sdS (128-byte swizzle, chunks of 8 queries)
            uint8_t *ds_row = sdS + (hh * kCW / 64) * kBoxBytes;
            const int chunk0 = (hh * kCW % 64) / 8;
            const uint64_t sc2 = f2_pack(p.scale, p.scale);
#pragma unroll
            for (int c = 0; c < kChunks; c++) {
                uint32_t dr[32];
                tmem_ld32(tmem + 128 + lane_off + (uint32_t)(hh * kCW + c * 32), dr);
                tc_wait_ld();
#pragma unroll
                for (int ch = 0; ch < 4; ch++) {
                    uint32_t w[4];
#pragma unroll
                    for (int u = 0; u < 4; u++) {
                        const int e = ch * 8 + 2 * u;
                        const int cc = c * 32 + e;
                        // dS = P * (scale*dP - scale*D)
                        const uint64_t t2 = f2_fma(f2_pack(__uint_as_float(dr[e]), __uint_as_float(dr[e + 1])), sc2,
                                                   *reinterpret_cast<const uint64_t *>(nsd + cc));
                        float d0, d1;
                        f2_unpack(f2_mul(t2, pf[cc >> 1]), d0, d1);
                        w[u] = pack_bf16x2(d0, d1);
                    }
                    *reinterpret_cast<uint4 *>(ds_row + swz128(r, chunk0 + c * 4 + ch)) =
                        make_uint4(w[0], w[1], w[2], w[3]);
                }
            }
            tc_wait_st();
            fence_proxy_async();  // dS^T stores -> visible to the tensor core's reads
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tl->ds_ready);
            // dQ^T(t): lane r is head dim r, columns my 64 queries
            if (!warp_wait(&tl->dq_full, t & 1, &tl->abort)) {
                set_timeout(tl, p.status);
                break;
            }
            tc_fence_after();
            uint32_t qa[kCW];
#pragma unroll
            for (int c = 0; c < kChunks; c++) tmem_ld32(tmem + 128 + lane_off + (uint32_t)(hh * kCW + c * 32), qa + c * 32);
            tc_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tl->dq_free);
            // stage dQ(t): query rows of 128 fp32 head dims (a warp store covers 128 contiguous
            // bytes of one row), rows 0-63 in pair t's Q stage once dK(t) is done, rows 64-127 in
            // its dO stage once dV(t) is done, so that half of the stores overlap dV(t); rows
            // past Lq hold zeros (their P, hence dS, is 0)
            const bool low_rows = hh * kCW < 64;
            if (!(low_rows ? warp_wait(&tl->dk_done, t & 1, &tl->abort)
                           : warp_wait(&tl->qdo_empty[st], (t >> 1) & 1, &tl->abort))) {
                set_timeout(tl, p.status);
                break;
            }
            float *stg = reinterpret_cast<float *>(low_rows ? sQ + st * kTileBytes : sdO + st * kTileBytes) +
                         ((hh * kCW) & 63) * 128 + r;
#pragma unroll
            for (int c = 0; c < kCW; c++) stg[c * 128] = __uint_as_float(qa[c]);
            fence_proxy_async();  // the stores -> visible to the bulk copy's reads
            __syncwarp();
            if (lane == 0) mbar_arrive(&tl->dq_staged[st]);
            t++;
            advance(p, i, g);
        }
        n_steps = t;

        // dK, dV of this block: lane r = key, my 64 head dims.  The TMEM loads are
        // warp-collective (.sync.aligned): every lane issues them, and only the
        // stores of keys past Lk (a partial last block) are left out.
        if (__all_sync(0xffffffffu, !tl->abort) && warp_wait(&tl->acc_done, 0, &tl->abort)) {
            tc_fence_after();
            const bool store = key < p.Lk;
            const size_t row_off = ((size_t)kvrow * p.Lk + (store ? key : 0)) * 128 + hh * kCW;
#pragma unroll
            for (int m = 0; m < 2; m++) {
                uint16_t *dst = (m ? p.dk : p.dv) + row_off;
                const uint32_t col = (m ? 384u : 256u) + (uint32_t)(hh * kCW);
#pragma unroll
                for (int c = 0; c < kChunks; c++) {
                    uint32_t v[32];
                    if (n_steps > 0) {  // warp-uniform
                        tmem_ld32(tmem + lane_off + col + c * 32, v);
                        tc_wait_ld();
                    } else {
#pragma unroll
                        for (int e = 0; e < 32; e++) v[e] = 0u;
                    }
                    if (store) {
#pragma unroll
                        for (int e = 0; e < 32; e += 8) {
                            uint4 o4;
                            o4.x = pack_bf16x2(__uint_as_float(v[e + 0]), __uint_as_float(v[e + 1]));
                            o4.y = pack_bf16x2(__uint_as_float(v[e + 2]), __uint_as_float(v[e + 3]));
                            o4.z = pack_bf16x2(__uint_as_float(v[e + 4]), __uint_as_float(v[e + 5]));
                            o4.w = pack_bf16x2(__uint_as_float(v[e + 6]), __uint_as_float(v[e + 7]));
                            *reinterpret_cast<uint4 *>(dst + c * 32 + e) = o4;
                        }
                    }
                }
            }
        } else if (!tl->abort) {
            set_timeout(tl, p.status);
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kMmaWarp) tmem_dealloc(tmem, 512);
}

// One warp per query row (padding rows included).
__global__ void __launch_bounds__(256) bwd_prep_kernel(const BwdParams p) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long row = (long long)blockIdx.x * 8 + warp;  // (b*Hq + hq) * Lq_pad + r
    if (row >= (long long)p.B * p.Hq * p.Lq_pad) return;
    const int r = (int)(row % p.Lq_pad);
    const long long bh = row / p.Lq_pad;
    float dsum = 0.f;
    float nl2 = -CUDART_INF_F;
    if (r < p.Lq) {
        const size_t src = ((size_t)bh * p.Lq + r) * 128 + lane * 4;
        const uint2 o2 = *reinterpret_cast<const uint2 *>(p.o + src);
        const uint2 d2 = *reinterpret_cast<const uint2 *>(p.dout + src);
        dsum = __uint_as_float(o2.x << 16) * __uint_as_float(d2.x << 16) +
               __uint_as_float(o2.x & 0xFFFF0000u) * __uint_as_float(d2.x & 0xFFFF0000u) +
               __uint_as_float(o2.y << 16) * __uint_as_float(d2.y << 16) +
               __uint_as_float(o2.y & 0xFFFF0000u) * __uint_as_float(d2.y & 0xFFFF0000u);
        const float lse = p.lse[(size_t)bh * p.Lq + r];
        if (lse > -CUDART_INF_F) nl2 = -lse * 1.4426950408889634f;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) dsum += __shfl_xor_sync(0xffffffffu, dsum, o);
    if (lane == 0) {
        p.neg_sdelta[row] = r < p.Lq ? -p.scale * dsum : 0.f;
        p.neg_lse2[row] = nl2;
    }
    reinterpret_cast<float4 *>(p.dq_acc + row * 128)[lane] = make_float4(0.f, 0.f, 0.f, 0.f);
}

// dq = bf16(dQ accumulator), 4 elements per thread.
__global__ void __launch_bounds__(256) bwd_finalize_kernel(const BwdParams p) {
    const long long idx = (long long)blockIdx.x * 256 + threadIdx.x;  // over B*Hq*Lq*32
    if (idx >= (long long)p.B * p.Hq * p.Lq * 32) return;
    const long long row = idx >> 5;  // (b*Hq + hq) * Lq + r
    const int c4 = (int)(idx & 31);
    const long long bh = row / p.Lq;
    const int r = (int)(row % p.Lq);
    const float4 a = reinterpret_cast<const float4 *>(p.dq_acc + ((size_t)bh * p.Lq_pad + r) * 128)[c4];
    uint2 out;
    out.x = pack_bf16x2(a.x, a.y);
    out.y = pack_bf16x2(a.z, a.w);
    reinterpret_cast<uint2 *>(p.dq + (size_t)row * 128)[c4] = out;
}

}  // namespace

cudaError_t launch_backward(const BwdParams &p, const CUtensorMap &tq, const CUtensorMap &tdo,
                            const CUtensorMap &tk, const CUtensorMap &tv, cudaStream_t st) {
    const long long prep_rows = (long long)p.B * p.Hq * p.Lq_pad;
    bwd_prep_kernel<<<(unsigned)((prep_rows + 7) / 8), 256, 0, st>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(bwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    dim3 grid(p.nb * p.Hkv, p.B);
    bwd_kernel<<<grid, kThreads, kSmemBytes, st>>>(p, tq, tdo, tk, tv);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const long long fin = (long long)p.B * p.Hq * p.Lq * 32;
    bwd_finalize_kernel<<<(unsigned)((fin + 255) / 256), 256, 0, st>>>(p);
    return cudaGetLastError();
}

}  // namespace blasst
