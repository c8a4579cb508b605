// decode.cu -- split-KV decode with softmax-threshold block skipping (BLASST),
// and the lse combine of the splits.
//
// One CTA per (split, KV head, sequence).  The tile is the G query heads x Lq
// queries that share the KV head (G*Lq <= 8*NT rows).  KV blocks are 64 keys.
//
// Warp roles (192 threads):
//   warps 0-3  consumers: each owns 16 keys of every block.  S^T = K_j q^T on
//              the tensor cores (mma.sync m16n8k16, keys on M, query rows on
//              N), block row maxima exchanged through shared memory, the
//              tile-wide skip decision, then for kept blocks exp2 and
//              O^T += V_j^T P^T (P re-laid out in registers with movmatrix).
//              The exponentials and P.V of a block run DQ blocks after its
//              decision (its scores wait in a register queue), so the V load
//              that the decision starts overlaps the next blocks' S.
//   warp 4     K producer: TMA loads of K blocks into a ring, as far ahead as
//              the ring allows; K is read for every block.
//   warp 5     V producer: waits for each block's published decision and
//              issues the TMA load of V_j only for kept blocks.  The decision
//              is taken before any V traffic for the block (xllm-io paper
//              review, section 3 "decode kernel optimisation": V_j of pruned
//              blocks is never loaded; gist.science (de) section 3: batched,
//              conditional V loads after the key blocks).
//
// The running max per row restarts in every split; the first visited block
// of a split is always kept.  With split seeding, every split after the first
// instead starts from the row maxima of block 0 (one extra K block through the
// ring, no decision, no V) and has no forced first block.  Scores are handled
// in log2 units: s2 = (q.k) * scale * log2(e), compared with log2(lambda).
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <math_constants.h>

#include "internal.h"
#include "ptx.cuh"

namespace blasst {
namespace {

constexpr int kConsumerWarps = 4;
constexpr int kConsumerThreads = kConsumerWarps * 32;
constexpr int kThreads = kConsumerThreads + 64;
constexpr int kStageBytes = kDecodeBlockN * 128 * 2;  // 64 keys x 128 dims bf16
constexpr int kBoxBytes = kStageBytes / 2;             // 64 keys x 64 dims (one 128-byte swizzle box)
constexpr int kStatusTimeout = 1;
constexpr int kStatusBadPage = 2;  // a page index or sequence length out of range

struct DecodeSmemTail {
    uint64_t k_full[8];
    uint64_t k_empty[8];
    uint64_t v_full[8];
    uint64_t v_empty[8];
    float red[2][kConsumerWarps][16];  // 16-byte aligned: read as float4
    float lred[kConsumerWarps][16];
    float rred[kConsumerWarps][16];
    float mfin[16];
    int dec_count;
    int abort;
};

// FP8 K/V cache: a ring stage is one 128-byte-swizzled box of 64 keys x 128 e4m3 bytes, and each
// consumer warp converts its 16 keys to f16 in a private slice laid out like a bf16 tile's 16 rows
// (two 64-column boxes of 16 rows x 128 bytes): two K slices (block j+1 is converted while the
// warps meet for block j's decision) and one V slice.
constexpr int kStageBytesF8 = kDecodeBlockN * 128;
constexpr int kSliceBoxBytes = 16 * 128;
constexpr int kSliceBytes = 2 * kSliceBoxBytes;

template <int NK, int NV, bool CALIB, bool F8>
constexpr int decode_smem_bytes() {
    return (NK + (CALIB ? 0 : NV)) * (F8 ? kStageBytesF8 : kStageBytes) + (F8 ? 3 * kConsumerWarps * kSliceBytes : 0) +
           (int)sizeof(DecodeSmemTail) + kMaxBlocksPerSplit + 1024;
}

// Warp `warp`'s 16 keys of a TMA-staged e4m3 block -> f16 in its slice (see kSliceBytes).
// Lane: row lane/2 of the 16, 64 of the 128 columns.
__device__ __forceinline__ void convert_slice_f8(const uint8_t *stage, uint8_t *slice, int warp, int lane) {
    const int r = lane >> 1, h = lane & 1;
    const uint8_t *src = stage + (warp * 16 + r) * 128;
#pragma unroll
    for (int c = 0; c < 4; c++) {
        const int c8 = h * 4 + c;  // 16-byte chunk of e4m3: columns 16*c8 .. 16*c8 + 15
        const uint4 v = *reinterpret_cast<const uint4 *>(src + ((c8 ^ (r & 7)) << 4));
        uint4 a, b;
        e4m3x4_to_f16x4(v.x, a.x, a.y);
        e4m3x4_to_f16x4(v.y, a.z, a.w);
        e4m3x4_to_f16x4(v.z, b.x, b.y);
        e4m3x4_to_f16x4(v.w, b.z, b.w);
        const int f0 = 2 * c8, f1 = 2 * c8 + 1;  // 16-byte chunks of f16
        *reinterpret_cast<uint4 *>(slice + (f0 >> 3) * kSliceBoxBytes + swz128(r, f0 & 7)) = a;
        *reinterpret_cast<uint4 *>(slice + (f1 >> 3) * kSliceBoxBytes + swz128(r, f1 & 7)) = b;
    }
}

__device__ __forceinline__ void set_timeout(DecodeSmemTail *t, unsigned int *status) {
    t->abort = 1;
    if (status) atomicOr(status, kStatusTimeout);
}

// TMA coordinates (row, plane) of block blk of KV head hkv of sequence b.  A paged
// cache maps the block through the block table; a page out of range is reported and
// read as the plane past the end (the copy then fills zeros).
__device__ __forceinline__ int2 kv_block_coord(const DecodeParams &p, int b, int hkv, int blk) {
    if (!p.block_table) return make_int2(blk * kDecodeBlockN, b * p.Hkv + hkv);
    int page = __ldg(p.block_table + (size_t)b * p.nb + blk);
    if (page < 0 || page >= p.num_pages) {
        if (p.status) atomicOr(p.status, kStatusBadPage);
        page = p.num_pages;
    }
    return make_int2(0, page * p.Hkv + hkv);
}

template <int NT, int NK, int NV, bool CALIB, bool F8>
__global__ void __launch_bounds__(kThreads, (F8 && NT == 1) ? 2 : 1)
    decode_split_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap tmap_k,
                        const __grid_constant__ CUtensorMap tmap_v) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *kring = smem;
    constexpr int SB = F8 ? kStageBytesF8 : kStageBytes;  // bytes of one K or V ring stage
    uint8_t *vring = smem + NK * SB;
    uint8_t *slices = vring + (CALIB ? 0 : NV * SB);  // FP8: per consumer warp, two K slices, then the V slices
    DecodeSmemTail *tl = reinterpret_cast<DecodeSmemTail *>(slices + (F8 ? 3 * kConsumerWarps * kSliceBytes : 0));
    volatile uint8_t *dec = reinterpret_cast<volatile uint8_t *>(tl + 1);

    // CTA order: every (sequence, KV head)'s first split, then its last split, then the middle ones.
    // The first and last chunks hold the sink and the most recent keys, where kept blocks gather,
    // so the CTAs with the most V traffic start early and the tail of the grid is made of the rest.
    int split, hkv, b;
    {
        const int groups = p.Hkv * p.B;
        const int L = blockIdx.x;
        int grp;
        if (L < groups) {
            split = 0;
            grp = L;
        } else if (p.num_splits > 1 && L < 2 * groups) {
            split = p.num_splits - 1;
            grp = L - groups;
        } else {
            const int m = L - min(2, p.num_splits) * groups;
            split = 1 + m / groups;
            grp = m % groups;
        }
        hkv = grp % p.Hkv;
        b = grp / p.Hkv;
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // keys of this sequence: all Lk, or (paged) its own length, split the same way
    int Lk = p.Lk, nbs = p.nb, per_split = p.per_split;
    if (p.seq_lens) {
        Lk = __ldg(p.seq_lens + b);
        if (Lk < 0 || Lk > p.Lk) {
            if (threadIdx.x == 0 && p.status) atomicOr(p.status, kStatusBadPage);
            Lk = min(max(Lk, 0), p.Lk);
        }
        nbs = (Lk + kDecodeBlockN - 1) / kDecodeBlockN;
        per_split = (nbs + p.num_splits - 1) / p.num_splits;
    }
    const int j0 = split * per_split;
    const int j1 = min(nbs, j0 + per_split);
    const int nblk = max(0, j1 - j0);
    const int bh = b * p.Hkv + hkv;
    // ring entries: [block 0 (seed)], then the split's blocks j0 .. j1-1
    const int seed = (p.seed && split > 0 && nblk > 0) ? 1 : 0;
    const int nent = nblk + seed;

    if (threadIdx.x == 0) {
        for (int i = 0; i < NK; i++) {
            mbar_init(&tl->k_full[i], 1);
            mbar_init(&tl->k_empty[i], kConsumerWarps);
        }
        if (!CALIB) {
            for (int i = 0; i < NV; i++) {
                mbar_init(&tl->v_full[i], 1);
                mbar_init(&tl->v_empty[i], kConsumerWarps);
            }
        }
        tl->dec_count = 0;
        tl->abort = 0;
        fence_mbar_init();
    }
    __syncthreads();

    // ------------------------------------------------------------ K producer
    if (warp == kConsumerWarps) {
        if (lane != 0) return;
        tma_prefetch_desc(&tmap_k);
        int issued = 0;
        for (int e = 0; e < nent; e++) {
            const int slot = e % NK;
            if (e >= NK && !mbar_wait(&tl->k_empty[slot], ((e / NK) & 1) ^ 1, &tl->abort)) {
                set_timeout(tl, p.status);
                break;
            }
            const int blk = (seed && e == 0) ? 0 : j0 + e - seed;
            const int2 cr = kv_block_coord(p, b, hkv, blk);
            uint8_t *dst = kring + slot * SB;
            mbar_arrive_expect_tx(&tl->k_full[slot], SB);
            tma_load_3d(dst, &tmap_k, &tl->k_full[slot], 0, cr.x, cr.y);
            if (!F8) tma_load_3d(dst + kBoxBytes, &tmap_k, &tl->k_full[slot], 64, cr.x, cr.y);
            issued++;
        }
        if (tl->abort) {  // let copies in flight land before the CTA exits
            for (int jj = max(0, issued - NK); jj < issued; jj++) mbar_wait(&tl->k_full[jj % NK], (jj / NK) & 1, nullptr);
        }
        return;
    }
    // ------------------------------------------------------------ V producer
    if (warp == kConsumerWarps + 1) {
        if (CALIB || lane != 0) return;
        tma_prefetch_desc(&tmap_v);
        int vk = 0;
        for (int jj = 0; jj < nblk && !tl->abort; jj++) {
            long long t0 = clock64();
            while (*reinterpret_cast<volatile int *>(&tl->dec_count) <= jj) {
                if (tl->abort || clock64() - t0 > kWaitLimitCycles) {
                    set_timeout(tl, p.status);
                    break;
                }
            }
            if (tl->abort) break;
            __threadfence_block();
            if (!dec[jj]) continue;
            const int slot = vk % NV;
            if (vk >= NV && !mbar_wait(&tl->v_empty[slot], ((vk / NV) & 1) ^ 1, &tl->abort)) {
                set_timeout(tl, p.status);
                break;
            }
            const int2 cr = kv_block_coord(p, b, hkv, j0 + jj);
            uint8_t *dst = vring + slot * SB;
            mbar_arrive_expect_tx(&tl->v_full[slot], SB);
            tma_load_3d(dst, &tmap_v, &tl->v_full[slot], 0, cr.x, cr.y);
            if (!F8) tma_load_3d(dst + kBoxBytes, &tmap_v, &tl->v_full[slot], 64, cr.x, cr.y);
            vk++;
        }
        if (tl->abort) {
            for (int i = max(0, vk - NV); i < vk; i++) mbar_wait(&tl->v_full[i % NV], (i / NV) & 1, nullptr);
        }
        return;
    }

    // ------------------------------------------------------------- consumers
    const int g4 = lane >> 2, t4 = lane & 3;
    constexpr int NC = 8 * NT;  // padded tile rows (columns of S^T)
    const int qrow0 = (b * p.Hq + hkv * p.G) * p.Lq;  // flat row index of tile row 0

    // q^T as mma B fragments, for all 8 k-steps of d = 128
    uint32_t qf[8][NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; nt++) {
        const int n = nt * 8 + g4;
        const uint32_t *qr = reinterpret_cast<const uint32_t *>(p.q + (size_t)(qrow0 + min(n, p.R - 1)) * 128);
#pragma unroll
        for (int ks = 0; ks < 8; ks++) {
            qf[ks][nt][0] = n < p.R ? __ldg(qr + ks * 8 + t4) : 0u;
            qf[ks][nt][1] = n < p.R ? __ldg(qr + ks * 8 + 4 + t4) : 0u;
            if (F8) {  // the FP8 path multiplies in f16: q re-rounded from bf16 (exact in f16's normal range)
#pragma unroll
                for (int u = 0; u < 2; u++)
                    qf[ks][nt][u] = pack_f16x2(__uint_as_float(qf[ks][nt][u] << 16),
                                               __uint_as_float(qf[ks][nt][u] & 0xFFFF0000u));
            }
        }
    }
    // last visible key of each of my columns (col = nt*8 + 2*t4 + e)
    int lastk[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; nt++)
#pragma unroll
        for (int e = 0; e < 2; e++) {
            const int c = nt * 8 + 2 * t4 + e;
            const int pos = c % p.Lq;
            lastk[nt][e] = c >= p.R ? -1 : (p.causal ? pos + (Lk - p.Lq) : Lk - 1);
        }

    float Mall[NC];
#pragma unroll
    for (int c = 0; c < NC; c++) Mall[c] = -CUDART_INF_F;
    float o_acc[CALIB ? 1 : 8][NT][4];
    // lsum: exact fp32 partial row sums (for lse); lrnd: sums of the bf16-rounded
    // P that P.V uses (normalises O exactly)
    float lsum[NT][2], lrnd[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; nt++) {
        lsum[nt][0] = lsum[nt][1] = 0.f;
        lrnd[nt][0] = lrnd[nt][1] = 0.f;
        if (!CALIB)
#pragma unroll
            for (int mt = 0; mt < 8; mt++)
#pragma unroll
                for (int i = 0; i < 4; i++) o_acc[mt][nt][i] = 0.f;
    }

    bool seen = false;
    int kept_count = 0;
    uint32_t mask_word = 0;
    int mask_word_idx = -1;
    unsigned long long n_skip = 0;
    const float NEG_INF = -CUDART_INF_F;

    // Software pipeline: a block's decision is published (and its V load requested) DQ
    // blocks before its exponentials and P.V run, so the V load is in flight meanwhile.
    // The decided blocks wait in a small queue in registers (shifted statically).
    constexpr int DQ = NT == 1 ? 2 : 1;
    float qs[DQ][NT][4], qmo[DQ][NT][2], qmn[DQ][NT][2];
    bool qk[DQ];
#pragma unroll
    for (int d = 0; d < DQ; d++) qk[d] = false;
    // P.V of a kept block: rescale by the growth of the running max, P = 2^(s - M), O += P V
    auto pv_block = [&](const float (&hs)[NT][4], const float (&hmo)[NT][2], const float (&hmn)[NT][2]) {
        uint32_t pb[NT][2];
#pragma unroll
        for (int nt = 0; nt < NT; nt++) {
            float pv[4];
#pragma unroll
            for (int e2 = 0; e2 < 2; e2++) {
                const float mold = hmo[nt][e2], mnew = hmn[nt][e2];
                const float alpha = (mnew == NEG_INF) ? 1.f : ex2(mold - mnew);
                lsum[nt][e2] *= alpha;
                lrnd[nt][e2] *= alpha;
#pragma unroll
                for (int mt = 0; mt < 8; mt++) {
                    o_acc[mt][nt][e2] *= alpha;
                    o_acc[mt][nt][2 + e2] *= alpha;
                }
                pv[e2] = hs[nt][e2] == NEG_INF ? 0.f : ex2(hs[nt][e2] - mnew);
                pv[2 + e2] = hs[nt][2 + e2] == NEG_INF ? 0.f : ex2(hs[nt][2 + e2] - mnew);
                lsum[nt][e2] += pv[e2] + pv[2 + e2];
            }
            uint32_t lo, hi;
            if constexpr (F8) {
                lo = pack_f16x2(pv[0], pv[1]);
                hi = pack_f16x2(pv[2], pv[3]);
                const float2 l2 = __half22float2(*reinterpret_cast<const __half2 *>(&lo));
                const float2 h2 = __half22float2(*reinterpret_cast<const __half2 *>(&hi));
                lrnd[nt][0] += l2.x + h2.x;
                lrnd[nt][1] += l2.y + h2.y;
            } else {
                lo = pack_bf16x2(pv[0], pv[1]);
                hi = pack_bf16x2(pv[2], pv[3]);
                lrnd[nt][0] += __uint_as_float(lo << 16) + __uint_as_float(hi << 16);
                lrnd[nt][1] += __uint_as_float(lo & 0xFFFF0000u) + __uint_as_float(hi & 0xFFFF0000u);
            }
            pb[nt][0] = movmatrix_t(lo);
            pb[nt][1] = movmatrix_t(hi);
        }
        const int vslot = kept_count % NV;
        if (!mbar_wait(&tl->v_full[vslot], (kept_count / NV) & 1, &tl->abort)) set_timeout(tl, p.status);
        const uint8_t *vb = vring + vslot * SB;
        if constexpr (F8) {
            uint8_t *vs = slices + (2 * kConsumerWarps + warp) * kSliceBytes;
            __syncwarp();  // the previous block's ldmatrix reads of this slice are done
            convert_slice_f8(vb, vs, warp, lane);
            __syncwarp();
            if (lane == 0) mbar_arrive(&tl->v_empty[vslot]);  // the stage is free once converted
            const int mi = lane >> 3, ri = lane & 7;
            const int r = ri + 8 * (mi >> 1);
#pragma unroll
            for (int mt = 0; mt < 8; mt++) {
                const int chunk = mt * 2 + (mi & 1);
                uint32_t a[4];
                ldsm_x4_t(smem_addr(vs + (chunk >> 3) * kSliceBoxBytes + swz128(r, chunk & 7)), a[0], a[1], a[2], a[3]);
#pragma unroll
                for (int nt = 0; nt < NT; nt++) mma_f16_16816(o_acc[mt][nt], a, pb[nt]);
            }
        } else {
            const int mi = lane >> 3, ri = lane & 7;
            const int key = warp * 16 + ri + 8 * (mi >> 1);
#pragma unroll
            for (int mt = 0; mt < 8; mt++) {
                const int chunk = mt * 2 + (mi & 1);
                uint32_t a[4];
                ldsm_x4_t(smem_addr(vb + (chunk >> 3) * kBoxBytes + swz128(key, chunk & 7)), a[0], a[1], a[2], a[3]);
#pragma unroll
                for (int nt = 0; nt < NT; nt++) mma_bf16_16816(o_acc[mt][nt], a, pb[nt]);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&tl->v_empty[vslot]);
        }
        kept_count++;
    };
    // queue a decided block, and run P.V for the oldest one if it was kept
    auto push_pop = [&](bool ck, const float (&cs)[NT][4], const float (&cmo)[NT][2], const float (&cmn)[NT][2]) {
        const bool hk = qk[0];
        float hs[NT][4], hmo[NT][2], hmn[NT][2];
#pragma unroll
        for (int nt = 0; nt < NT; nt++) {
#pragma unroll
            for (int i = 0; i < 4; i++) hs[nt][i] = qs[0][nt][i];
#pragma unroll
            for (int i = 0; i < 2; i++) {
                hmo[nt][i] = qmo[0][nt][i];
                hmn[nt][i] = qmn[0][nt][i];
            }
        }
#pragma unroll
        for (int d = 0; d + 1 < DQ; d++) {
            qk[d] = qk[d + 1];
#pragma unroll
            for (int nt = 0; nt < NT; nt++) {
#pragma unroll
                for (int i = 0; i < 4; i++) qs[d][nt][i] = qs[d + 1][nt][i];
#pragma unroll
                for (int i = 0; i < 2; i++) {
                    qmo[d][nt][i] = qmo[d + 1][nt][i];
                    qmn[d][nt][i] = qmn[d + 1][nt][i];
                }
            }
        }
        qk[DQ - 1] = ck;
#pragma unroll
        for (int nt = 0; nt < NT; nt++) {
#pragma unroll
            for (int i = 0; i < 4; i++) qs[DQ - 1][nt][i] = cs[nt][i];
#pragma unroll
            for (int i = 0; i < 2; i++) {
                qmo[DQ - 1][nt][i] = cmo[nt][i];
                qmn[DQ - 1][nt][i] = cmn[nt][i];
            }
        }
        if (hk) pv_block(hs, hmo, hmn);
    };

    // FP8: K of ring entry e -> this warp's K slice e & 1, then the ring stage goes back
    auto convert_k = [&](int e) {
        const int ns = e % NK;
        if (!mbar_wait(&tl->k_full[ns], (e / NK) & 1, &tl->abort)) set_timeout(tl, p.status);
        __syncwarp();  // the slice's previous ldmatrix reads are done
        convert_slice_f8(kring + ns * SB, slices + (warp * 2 + (e & 1)) * kSliceBytes, warp, lane);
        __syncwarp();
        if (lane == 0) mbar_arrive(&tl->k_empty[ns]);
    };
    if constexpr (F8) {
        if (nent > 0) convert_k(0);
    }

    for (int e = 0; e < nent; e++) {
        const int jj = e - seed;  // block index within the split; -1: the seed block
        const int j = jj < 0 ? 0 : j0 + jj;
        const int slot = e % NK;
        if (!F8 && !mbar_wait(&tl->k_full[slot], (e / NK) & 1, &tl->abort)) set_timeout(tl, p.status);
        const uint8_t *kb = kring + slot * SB;

        // two independent accumulation chains (even and odd 16-column steps of d), added at the
        // end: half the dependent mma latency per block
        float acc[NT][4], acc2[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; nt++)
#pragma unroll
            for (int i = 0; i < 4; i++) acc[nt][i] = acc2[nt][i] = 0.f;
        if constexpr (F8) {
            const uint8_t *ks_ = slices + (warp * 2 + (e & 1)) * kSliceBytes;  // converted ahead
            const int mi = lane >> 3, ri = lane & 7;
            const int r = ri + 8 * (mi & 1);
#pragma unroll
            for (int ks = 0; ks < 8; ks++) {
                const int chunk = ks * 2 + (mi >> 1);
                uint32_t a[4];
                ldsm_x4(smem_addr(ks_ + (chunk >> 3) * kSliceBoxBytes + swz128(r, chunk & 7)), a[0], a[1], a[2], a[3]);
#pragma unroll
                for (int nt = 0; nt < NT; nt++) mma_f16_16816((ks & 1) ? acc2[nt] : acc[nt], a, qf[ks][nt]);
            }
        } else {
            const int mi = lane >> 3, ri = lane & 7;
            const int key = warp * 16 + ri + 8 * (mi & 1);
#pragma unroll
            for (int ks = 0; ks < 8; ks++) {
                const int chunk = ks * 2 + (mi >> 1);
                uint32_t a[4];
                ldsm_x4(smem_addr(kb + (chunk >> 3) * kBoxBytes + swz128(key, chunk & 7)), a[0], a[1], a[2], a[3]);
#pragma unroll
                for (int nt = 0; nt < NT; nt++) mma_bf16_16816((ks & 1) ? acc2[nt] : acc[nt], a, qf[ks][nt]);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&tl->k_empty[slot]);
        }
#pragma unroll
        for (int nt = 0; nt < NT; nt++)
#pragma unroll
            for (int i = 0; i < 4; i++) acc[nt][i] += acc2[nt][i];

        // scaled, masked scores in log2 units; my keys: lo = g4, hi = g4 + 8
        const int key_lo = j * kDecodeBlockN + warp * 16 + g4;
        float s[NT][4];
        float cmax[NT][2];
#pragma unroll
        for (int nt = 0; nt < NT; nt++) {
#pragma unroll
            for (int e = 0; e < 2; e++) {
                s[nt][e] = key_lo <= lastk[nt][e] && key_lo < Lk ? acc[nt][e] * p.scale_log2 : NEG_INF;
                s[nt][2 + e] = key_lo + 8 <= lastk[nt][e] && key_lo + 8 < Lk ? acc[nt][2 + e] * p.scale_log2 : NEG_INF;
                float m = fmaxf(s[nt][e], s[nt][2 + e]);
                m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 4));
                m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 8));
                m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 16));
                cmax[nt][e] = m;
            }
        }
        if (g4 == 0) {
#pragma unroll
            for (int nt = 0; nt < NT; nt++) {
                tl->red[e & 1][warp][nt * 8 + 2 * t4] = cmax[nt][0];
                tl->red[e & 1][warp][nt * 8 + 2 * t4 + 1] = cmax[nt][1];
            }
        }
        if constexpr (F8) {
            if (e + 1 < nent) convert_k(e + 1);  // overlaps the other warps reaching the barrier
        }
        asm volatile("bar.sync 1, %0;" ::"n"(kConsumerThreads) : "memory");

        if (jj < 0) {
            // the seed block: its row maxima start the running max of this split
#pragma unroll
            for (int c = 0; c < NC; c++) {
                float mt = tl->red[e & 1][0][c];
#pragma unroll
                for (int w = 1; w < kConsumerWarps; w++) mt = fmaxf(mt, tl->red[e & 1][w][c]);
                Mall[c] = mt;
            }
            seen = true;  // no forced first block after a seed
            continue;
        }

        // block row maxima of the whole tile (four warps' partial maxima, read as float4),
        // running max after the block, gap
        float mtc[NC];
#pragma unroll
        for (int c4 = 0; c4 < NC / 4; c4++) {
            float4 v = *reinterpret_cast<const float4 *>(&tl->red[e & 1][0][4 * c4]);
#pragma unroll
            for (int w = 1; w < kConsumerWarps; w++) {
                const float4 u = *reinterpret_cast<const float4 *>(&tl->red[e & 1][w][4 * c4]);
                v.x = fmaxf(v.x, u.x);
                v.y = fmaxf(v.y, u.y);
                v.z = fmaxf(v.z, u.z);
                v.w = fmaxf(v.w, u.w);
            }
            mtc[4 * c4] = v.x;
            mtc[4 * c4 + 1] = v.y;
            mtc[4 * c4 + 2] = v.z;
            mtc[4 * c4 + 3] = v.w;
        }
        float Mn[NC];
        float gap = NEG_INF;
        bool visited = false;
#pragma unroll
        for (int c = 0; c < NC; c++) {
            const float mt = mtc[c];
            Mn[c] = fmaxf(Mall[c], mt);
            if (mt > NEG_INF) {
                visited = true;
                gap = fmaxf(gap, mt - Mn[c]);
            }
        }
        const bool first = visited && !seen;
        seen = seen || visited;
        const bool skip = visited && !first && (gap < p.thr_log2);
        const bool kept = visited && !skip;

        if (warp == 0 && lane == 0) {
            if (!CALIB) {
                dec[jj] = kept ? 1 : 0;
                __threadfence_block();
                *reinterpret_cast<volatile int *>(&tl->dec_count) = jj + 1;
            }
            if (p.gaps)
                p.gaps[(size_t)bh * p.nb + j] =
                    !visited ? CUDART_NAN_F : (first ? CUDART_INF_F : gap * 0.69314718055994531f);
            if (skip) {
                n_skip++;
                if (p.skip_mask) {
                    if (mask_word_idx != (j >> 5)) {
                        if (mask_word_idx >= 0 && mask_word)
                            atomicOr(p.skip_mask + (size_t)bh * p.words + mask_word_idx, mask_word);
                        mask_word_idx = j >> 5;
                        mask_word = 0;
                    }
                    mask_word |= 1u << (j & 31);
                }
            }
        }
        if constexpr (CALIB) {
            if (kept) {
#pragma unroll
                for (int c = 0; c < NC; c++) Mall[c] = Mn[c];
            }
        } else {
        // queue the block: its scores and, for my columns, the running max before and after it
        float cs[NT][4], cmo[NT][2], cmn[NT][2];
#pragma unroll
        for (int nt = 0; nt < NT; nt++)
#pragma unroll
            for (int e2 = 0; e2 < 2; e2++) {
                const int c = nt * 8 + 2 * t4 + e2;
                float mold = NEG_INF, mnew = NEG_INF;
#pragma unroll
                for (int cc = 0; cc < NC; cc++)
                    if (cc == c) {
                        mold = Mall[cc];
                        mnew = Mn[cc];
                    }
                cmo[nt][e2] = mold;
                cmn[nt][e2] = mnew;
                cs[nt][e2] = s[nt][e2];
                cs[nt][2 + e2] = s[nt][2 + e2];
            }
        if (kept) {
#pragma unroll
            for (int c = 0; c < NC; c++) Mall[c] = Mn[c];
        }
        push_pop(kept, cs, cmo, cmn);
        }
    }
    if constexpr (!CALIB) {
        // the last queued blocks
        float zs[NT][4] = {}, zm[NT][2] = {};
#pragma unroll
        for (int d = 0; d < DQ; d++) push_pop(false, zs, zm, zm);
    }

    if (warp == 0 && lane == 0) {
        if (p.skip_mask && mask_word_idx >= 0 && mask_word)
            atomicOr(p.skip_mask + (size_t)bh * p.words + mask_word_idx, mask_word);
        if (p.split_skips)
            p.split_skips[blockIdx.x] = (unsigned int)n_skip;
        else if (p.skip_count && n_skip)
            atomicAdd(p.skip_count, n_skip);
    }
    if (CALIB) return;

    // ------------------------------------------------ reduce over the 4 warps
    // partial O^T of each warp -> shared memory (the K ring is idle now)
    float *obuf = reinterpret_cast<float *>(kring);  // [warp][dv 128][NC]
#pragma unroll
    for (int nt = 0; nt < NT; nt++) {
#pragma unroll
        for (int e = 0; e < 2; e++) {
            float l = lsum[nt][e], lr = lrnd[nt][e];
#pragma unroll
            for (int o = 4; o < 32; o <<= 1) {
                l += __shfl_xor_sync(0xffffffffu, l, o);
                lr += __shfl_xor_sync(0xffffffffu, lr, o);
            }
            if (g4 == 0) {
                tl->lred[warp][nt * 8 + 2 * t4 + e] = l;
                tl->rred[warp][nt * 8 + 2 * t4 + e] = lr;
            }
        }
#pragma unroll
        for (int mt = 0; mt < 8; mt++) {
            const int dv0 = mt * 16 + g4;
            const int c0 = nt * 8 + 2 * t4;
            obuf[(warp * 128 + dv0) * NC + c0] = o_acc[mt][nt][0];
            obuf[(warp * 128 + dv0) * NC + c0 + 1] = o_acc[mt][nt][1];
            obuf[(warp * 128 + dv0 + 8) * NC + c0] = o_acc[mt][nt][2];
            obuf[(warp * 128 + dv0 + 8) * NC + c0 + 1] = o_acc[mt][nt][3];
        }
    }
    if (threadIdx.x == 0) {
#pragma unroll
        for (int c = 0; c < NC; c++) tl->mfin[c] = Mall[c];
    }
    asm volatile("bar.sync 1, %0;" ::"n"(kConsumerThreads) : "memory");

    const int x = threadIdx.x;  // dv index 0..127
    const int S = p.num_splits;
    for (int c = 0; c < p.R; c++) {
        float l = 0.f, lr = 0.f, o = 0.f;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; w++) {
            l += tl->lred[w][c];
            lr += tl->rred[w][c];
            o += obuf[(w * 128 + x) * NC + c];
        }
        const size_t row = (size_t)(qrow0 + c) * S + split;
        p.part_o[row * 128 + x] = lr > 0.f ? (F8 ? p.v_scale : 1.f) * o / lr : 0.f;
        if (x == 0) p.part_lse[row] = l > 0.f ? (tl->mfin[c] + __log2f(l)) * 0.69314718055994531f : NEG_INF;
    }
}

// One warp per output row: lse = ln sum_s exp(lse_s); O = sum_s exp(lse_s - lse) O_s.
__global__ void __launch_bounds__(128) combine_kernel(const CombineParams p) {
    pdl_wait();  // the split kernel has finished and its partials are visible
    const int row = blockIdx.x * 4 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (p.skip_count && blockIdx.x == 0) {
        // the split CTAs' skip counts, one slot each: their sum is the call's count
        __shared__ unsigned long long part[4];
        unsigned long long s = 0;
        for (int i = threadIdx.x; i < p.n_counts; i += 128) s += p.split_skips[i];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if (lane == 0) part[threadIdx.x >> 5] = s;
        __syncthreads();
        if (threadIdx.x == 0) *p.skip_count = part[0] + part[1] + part[2] + part[3];
    }
    if (row >= p.rows) return;
    const int S = p.num_splits;
    const float LOG2E = 1.4426950408889634f;
    float mx = -CUDART_INF_F;
    for (int s = lane; s < S; s += 32) mx = fmaxf(mx, p.part_lse[(size_t)row * S + s]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float sum = 0.f;
    if (mx > -CUDART_INF_F)
        for (int s = lane; s < S; s += 32) sum += ex2((p.part_lse[(size_t)row * S + s] - mx) * LOG2E);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    const float L = mx > -CUDART_INF_F ? mx + __logf(sum) : -CUDART_INF_F;
    for (int x0 = lane * 4; x0 < p.dv; x0 += 128) {
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        if (L > -CUDART_INF_F) {
            for (int s = 0; s < S; s++) {
                const float ls = p.part_lse[(size_t)row * S + s];
                if (ls == -CUDART_INF_F) continue;
                const float w = ex2((ls - L) * LOG2E);
                const float4 v = *reinterpret_cast<const float4 *>(p.part_o + ((size_t)row * S + s) * p.dv + x0);
                acc[0] += w * v.x;
                acc[1] += w * v.y;
                acc[2] += w * v.z;
                acc[3] += w * v.w;
            }
        }
        uint2 packed;
        packed.x = pack_bf16x2(acc[0], acc[1]);
        packed.y = pack_bf16x2(acc[2], acc[3]);
        *reinterpret_cast<uint2 *>(p.o + (size_t)row * p.dv + x0) = packed;
    }
    if (lane == 0) p.lse[row] = L;
}

template <int NT, bool CALIB, bool F8 = false>
cudaError_t launch_decode_t(const DecodeParams &p, const CUtensorMap &tk, const CUtensorMap &tv, cudaStream_t st) {
    constexpr int NK = 4, NV = 2;
    constexpr int smem = decode_smem_bytes<NK, NV, CALIB, F8>();
    auto kern = decode_split_kernel<NT, NK, NV, CALIB, F8>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    kern<<<p.num_splits * p.Hkv * p.B, kThreads, smem, st>>>(p, tk, tv);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode(const DecodeParams &p, const CUtensorMap &tk, const CUtensorMap &tv, bool calib, int nt,
                          cudaStream_t st) {
    if (calib) return nt == 1 ? launch_decode_t<1, true>(p, tk, tv, st) : launch_decode_t<2, true>(p, tk, tv, st);
    return nt == 1 ? launch_decode_t<1, false>(p, tk, tv, st) : launch_decode_t<2, false>(p, tk, tv, st);
}

cudaError_t launch_decode_fp8(const DecodeParams &p, const CUtensorMap &tk, const CUtensorMap &tv, int nt,
                              cudaStream_t st) {
    return nt == 1 ? launch_decode_t<1, false, true>(p, tk, tv, st) : launch_decode_t<2, false, true>(p, tk, tv, st);
}

cudaError_t launch_combine(const CombineParams &p, cudaStream_t st) {
    if (p.rows == 0) return cudaSuccess;
    // programmatic dependent launch: the combine's launch is processed while the split
    // kernel runs, and its CTAs start as the split CTAs exit, each waiting on the device
    // (griddepcontrol.wait) for the split grid's completion and memory.  (An explicit early
    // signal from the split CTAs, at their start, measured slower.)
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((p.rows + 3) / 4);
    cfg.blockDim = dim3(128);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, combine_kernel, p);
}

}  // namespace blasst
