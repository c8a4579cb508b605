// internal.h -- parameters shared between the C-ABI host layer and the kernels.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/blasst.h"

namespace blasst {

constexpr int kDecodeBlockN = 64;
constexpr int kPrefillBlockM = 128;
constexpr int kPrefillBlockN = 128;
constexpr int kMaxBlocksPerSplit = 8192;

// One decode (or decode-shaped calibration) call.
struct DecodeParams {
    const uint16_t *q;              // [B, Hq, Lq, d] bf16
    float *part_o;                  // [B*Hq*Lq, S, dv] fp32 split outputs (normalised)
    float *part_lse;                // [B*Hq*Lq, S] fp32 split lse (natural log)
    uint32_t *skip_mask;            // [B, Hkv, 1, W] or null
    unsigned long long *skip_count; // or null: every CTA adds its skipped blocks (calibration pass)
    unsigned int *split_skips;      // or null: every CTA stores its skipped blocks in its own slot
                                    // (attention calls; the combine kernel sums the slots)
    float *gaps;                    // [B*Hkv, nb] or null
    unsigned int *status;           // or null
    int B, Hq, Hkv, Lq, Lk, G, R;   // R = G * Lq rows per tile
    int nb, num_splits, per_split, words;
    int causal;
    float scale_log2;               // scale * log2(e)
    float thr_log2;                 // log2(lambda), -inf for lambda = 0
    int seed;                       // 1: splits after the first start from block 0's row maxima
    float v_scale;                  // FP8 cache: V = v_scale * e4m3 (scale_log2 already holds k_scale)
    // paged cache (null: contiguous): K/V pages [num_pages, Hkv, 64, 128]; sequence b has
    // seq_lens[b] keys in pages block_table[b * nb + i]; Lk and nb are then the maxima
    const int *block_table;
    const int *seq_lens;
    int num_pages;
};

struct CombineParams {
    const float *part_o;
    const float *part_lse;
    uint16_t *o;      // [B, Hq, Lq, dv] bf16
    float *lse;       // [B, Hq, Lq]
    int rows;         // B * Hq * Lq
    int num_splits;
    int dv;
    const unsigned int *split_skips;  // per-CTA skip counts of the split kernel, or null
    int n_counts;                     // slots in split_skips
    unsigned long long *skip_count;   // their sum is stored here (when not null)
};

// One prefill (or prefill-shaped calibration) call.
struct PrefillParams {
    uint16_t *o;                    // [B, Hq, Lq, 128] bf16
    float *lse;                     // [B, Hq, Lq]
    uint32_t *skip_mask;            // [B, Hq, n_qtiles, W] or null
    unsigned long long *skip_count; // or null
    float *gaps;                    // [B*Hq*n_qtiles, nb] or null
    unsigned int *status;           // or null
    int B, Hq, Hkv, Lq, Lk, G;
    int n_qtiles, nb, words;
    int causal;
    float scale_log2;
    float thr_log2;
};

// One fixed-mask backward call (prefill tiling: 128-row query tiles, 128-key blocks, d = 128).
struct BwdParams {
    const uint16_t *o;              // [B, Hq, Lq, 128] bf16 forward output
    const uint16_t *dout;           // [B, Hq, Lq, 128] bf16 upstream gradient
    const float *lse;               // [B, Hq, Lq] forward lse (natural log)
    float *neg_lse2;                // workspace [B*Hq, Lq_pad]: -lse*log2(e), -inf on padding rows
    float *neg_sdelta;              // workspace [B*Hq, Lq_pad]: -scale * rowsum(dO * O)
    float *dq_acc;                  // workspace [B*Hq, Lq_pad, 128] fp32
    uint16_t *dq;                   // [B, Hq, Lq, 128] bf16
    uint16_t *dk, *dv;              // [B, Hkv, Lk, 128] bf16
    const uint32_t *skip_mask;      // [B, Hq, nq, words] from the forward, or null (nothing skipped)
    unsigned int *status;           // or null
    int B, Hq, Hkv, Lq, Lk, G, Lq_pad, nq, nb, words, causal;
    float scale_log2;               // scale * log2(e)
    float scale;
};
// One MLA decode (or MLA-shaped calibration) call: a single latent KV head of
// 576 columns, V = its first 512 columns.
struct MlaParams {
    const uint16_t *q;              // [B, Hq*Lq, 576] bf16 queries (dense rows)
    float *part_o;                  // [B*Hq*Lq, S, 512] fp32 split outputs (normalised)
    float *part_lse;                // [B*Hq*Lq, S]
    uint32_t *skip_mask;            // [B, 1, 1, W] or null
    unsigned long long *skip_count; // or null (calibration pass: added to)
    unsigned int *split_skips;      // [B, S] or null (attention calls: one slot per split)
    float *gaps;                    // [B, nb] or null
    unsigned int *status;           // or null
    int B, Hq, Lq, Lk, R;           // R = Hq * Lq <= 128
    int nb, num_splits, per_split, words;
    int causal;
    float scale_log2;
    float thr_log2;
    int seed;                       // 1: splits after the first start from block 0's row maxima
};

// prep (delta, lse2, zeroed dQ accumulator), the main tcgen05 kernel, dq finalize
cudaError_t launch_backward(const BwdParams &p, const CUtensorMap &tmap_q, const CUtensorMap &tmap_do,
                            const CUtensorMap &tmap_k, const CUtensorMap &tmap_v, cudaStream_t stream);
// Records the text returned by blasst_last_error() for this thread.
void set_last_error(const char *msg);
// The split count a decode call with these arguments uses (rows = G * Lq, the tile's rows):
// num_splits when positive; 0 -> 16 (d = 128) or 2 (MLA, d = 576); -1 ->
// blasst_decode_pick_splits_rows with the current device's SM count (d = 128 only;
// BLASST_ERR_INVALID for MLA and other negative values).
blasst_status decode_split_count(int d, int num_splits, int B, int Hkv, int rows, int Lk, int *out);

cudaError_t launch_decode(const DecodeParams &p, const CUtensorMap &tmap_k, const CUtensorMap &tmap_v, bool calib,
                          int nt, cudaStream_t stream);
// FP8 (e4m3) K/V cache, d = 128, tiles of up to 16 rows; tmaps are u8 boxes of 128 x 64
cudaError_t launch_decode_fp8(const DecodeParams &p, const CUtensorMap &tmap_k, const CUtensorMap &tmap_v, int nt,
                              cudaStream_t stream);
cudaError_t launch_combine(const CombineParams &p, cudaStream_t stream);
// Decode tiles of 17..128 rows (d = 128) on tcgen05; tmap_q covers q as [B][Hq*Lq][128].
cudaError_t launch_decode_wide(const DecodeParams &p, const CUtensorMap &tmap_q, const CUtensorMap &tmap_k,
                               const CUtensorMap &tmap_v, bool calib, cudaStream_t stream);
cudaError_t launch_mla(const MlaParams &p, const CUtensorMap &tmap_q, const CUtensorMap &tmap_k, bool calib,
                       cudaStream_t stream);
cudaError_t launch_prefill(const PrefillParams &p, const CUtensorMap &tmap_q, const CUtensorMap &tmap_k,
                           const CUtensorMap &tmap_v, bool calib, cudaStream_t stream);
// The prefill with the skip decision compiled out (measurement instance; never used by the API).
cudaError_t launch_prefill_novote(const PrefillParams &p, const CUtensorMap &tmap_q, const CUtensorMap &tmap_k,
                                  const CUtensorMap &tmap_v, cudaStream_t stream);

}  // namespace blasst
