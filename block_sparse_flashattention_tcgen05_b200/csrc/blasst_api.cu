// blasst_api.cu -- the extern "C" boundary of libblasst.so: argument checks,
// TMA descriptors, workspace, and the kernel launches.  No compute here.
#include <algorithm>
#include <cmath>
#include <cstdio>
#include <climits>
#include <cstring>
#include <vector>

#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/blasst.h"
#include "../../include/blasst_measure.h"
#include "internal.h"

using namespace blasst;

namespace {
thread_local char g_last_error[256] = "";
}  // namespace

void blasst::set_last_error(const char *msg) { std::snprintf(g_last_error, sizeof g_last_error, "%s", msg); }

namespace {

blasst_status cuda_fail(cudaError_t e, const char *where) {
    std::snprintf(g_last_error, sizeof g_last_error, "%s: %s", where, cudaGetErrorString(e));
    return BLASST_ERR_CUDA;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static bool tried = false;
    if (!tried) {
        tried = true;
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    return fn;
}

// 3-D bf16 view [outer, rows, cols] with row stride `row_stride` elements and
// outer stride rows*row_stride; box of box_cols x box_rows x 1, 128B swizzle.
blasst_status make_tmap(CUtensorMap *m, const void *base, long long cols, long long rows, long long outer,
                        long long row_stride, int box_cols, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) {
        std::snprintf(g_last_error, sizeof g_last_error, "cuTensorMapEncodeTiled unavailable");
        return BLASST_ERR_CUDA;
    }
    cuuint64_t dims[3] = {(cuuint64_t)cols, (cuuint64_t)rows, (cuuint64_t)outer};
    cuuint64_t strides[2] = {(cuuint64_t)row_stride * 2, (cuuint64_t)rows * row_stride * 2};
    cuuint32_t box[3] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        std::snprintf(g_last_error, sizeof g_last_error, "cuTensorMapEncodeTiled failed (%d)", (int)r);
        return BLASST_ERR_CUDA;
    }
    return BLASST_OK;
}

// 3-D view of an e4m3 (byte) cache [outer, rows, 128]: one 128-byte-swizzled box of 128 x box_rows.
blasst_status make_tmap_u8(CUtensorMap *m, const void *base, long long rows, long long outer, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) {
        std::snprintf(g_last_error, sizeof g_last_error, "cuTensorMapEncodeTiled unavailable");
        return BLASST_ERR_CUDA;
    }
    cuuint64_t dims[3] = {128, (cuuint64_t)rows, (cuuint64_t)outer};
    cuuint64_t strides[2] = {128, (cuuint64_t)rows * 128};
    cuuint32_t box[3] = {128, (cuuint32_t)box_rows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void *>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        std::snprintf(g_last_error, sizeof g_last_error, "cuTensorMapEncodeTiled failed (%d)", (int)r);
        return BLASST_ERR_CUDA;
    }
    return BLASST_OK;
}

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Copy of the caller's options with fields past struct_size zeroed.
blasst_opts read_opts(const blasst_opts *o) {
    blasst_opts r;
    std::memset(&r, 0, sizeof r);
    if (o) {
        size_t n = std::min(o->struct_size, sizeof r);
        if (n > 0) std::memcpy(&r, o, n);
    }
    r.struct_size = sizeof r;
    return r;
}

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

struct Common {
    int dv;
    long long krs, vrs;
};

blasst_status check_common(const void *q, const void *k, int B, int Hq, int Hkv, int Lq, int Lk, int d, float scale,
                           float lambda, int causal, const blasst_opts &o, Common *c) {
    if (!q || !k) return BLASST_ERR_INVALID;
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Lq <= 0 || Lk <= 0 || d <= 0) return BLASST_ERR_INVALID;
    if (Hq % Hkv != 0) return BLASST_ERR_INVALID;
    if (!(std::isfinite(scale) && scale > 0.f)) return BLASST_ERR_INVALID;
    if (!(std::isfinite(lambda) && lambda >= 0.f && lambda < 1.f)) return BLASST_ERR_INVALID;
    if (causal && Lq > Lk) return BLASST_ERR_INVALID;
    if (!aligned(q, 16) || !aligned(k, 16)) return BLASST_ERR_INVALID;
    c->dv = o.dv ? o.dv : d;
    c->krs = o.k_row_stride ? o.k_row_stride : d;
    c->vrs = o.v_row_stride ? o.v_row_stride : c->dv;
    if (c->dv <= 0 || c->krs < d || c->vrs < c->dv || c->krs % 8 || c->vrs % 8) return BLASST_ERR_INVALID;
    if (o.workspace && !aligned(o.workspace, 256)) return BLASST_ERR_INVALID;
    return BLASST_OK;
}

float log2_threshold(float lambda) {
    return lambda > 0.f ? (float)(std::log((double)lambda) / std::log(2.0)) : -INFINITY;
}

const double kLog2e = 1.4426950408889634;

}  // namespace

blasst_status blasst::decode_split_count(int d, int num_splits, int B, int Hkv, int rows, int Lk, int *out) {
    *out = 0;
    if (num_splits > 0) {
        *out = num_splits;
        return BLASST_OK;
    }
    if (num_splits == 0) {
        *out = d == 576 ? 2 : 16;  // MLA: two CTAs per split already fill the device at batch 64
        return BLASST_OK;
    }
    if (num_splits != -1 || d == 576) return BLASST_ERR_INVALID;
    // adaptive: from the batch, the cache length and this device's SM count
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute(multiprocessors)");
    *out = blasst_decode_pick_splits_rows(B, Hkv, rows, Lk, sms);
    return BLASST_OK;
}

namespace {

// ---------------------------------------------------------------------- MLA
blasst_status run_mla(const void *q, const void *k, const void *v, void *o, float *lse, int B, int Hq, int Hkv,
                      int Lq, int Lk, int d, float scale, float lambda, int causal, uint32_t *skip_mask,
                      unsigned long long *skip_count, void *stream, const blasst_opts &op, const Common &c,
                      bool calib) {
    // one latent KV head; V = the first 512 columns of the same cache rows
    if (Hkv != 1 || c.dv != 512 || c.krs != d) return BLASST_ERR_UNSUPPORTED;
    if (!calib && (v != k || c.vrs != c.krs)) return BLASST_ERR_UNSUPPORTED;
    const long long R = (long long)Hq * Lq;
    if (R > 128) return BLASST_ERR_UNSUPPORTED;
    int S = 0;
    blasst_status sst = decode_split_count(d, op.num_splits, B, Hkv, (int)R, Lk, &S);
    if (sst != BLASST_OK) return sst;
    if (S > 65535 || B > 65535) return BLASST_ERR_INVALID;
    const int nb = (Lk + kDecodeBlockN - 1) / kDecodeBlockN;
    const int per_split = (nb + S - 1) / S;
    const int words = (nb + 31) / 32;
    const size_t rows = (size_t)B * Hq * Lq;
    const size_t need = blasst_decode_workspace_bytes(B, Hq, Lq, c.dv, S);
    void *ws = op.workspace;
    if (!calib && ws && op.workspace_bytes < need) return BLASST_ERR_WORKSPACE;
    cudaStream_t sm = reinterpret_cast<cudaStream_t>(stream);

    CUtensorMap tq, tk;
    blasst_status st = make_tmap(&tq, q, d, R, B, d, 64, 128);
    if (st != BLASST_OK) return st;
    st = make_tmap(&tk, k, d, Lk, B, c.krs, 64, kDecodeBlockN);
    if (st != BLASST_OK) return st;
    bool own_ws = false;
    cudaError_t e;
    if (!calib && !ws) {
        e = cudaMallocAsync(&ws, need, sm);
        if (e != cudaSuccess) return cuda_fail(e, "cudaMallocAsync(workspace)");
        own_ws = true;
    }
    if (skip_mask) {
        e = cudaMemsetAsync(skip_mask, 0, (size_t)B * words * sizeof(uint32_t), sm);
        if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(skip_mask)");
    }
    // the calibration pass adds into skip_count; an attention call's split CTAs store their
    // counts in the workspace and the combine kernel writes the sum (no reset needed)
    if (skip_count && calib) {
        e = cudaMemsetAsync(skip_count, 0, sizeof(unsigned long long), sm);
        if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(skip_count)");
    }
    MlaParams p;
    std::memset(&p, 0, sizeof p);
    p.q = static_cast<const uint16_t *>(q);
    p.part_o = calib ? nullptr : static_cast<float *>(ws);
    p.part_lse = calib ? nullptr : reinterpret_cast<float *>(static_cast<char *>(ws) + round_up(rows * S * c.dv * 4, 256));
    p.skip_mask = skip_mask;
    p.skip_count = calib ? skip_count : nullptr;
    p.split_skips = (calib || !skip_count) ? nullptr
                                           : reinterpret_cast<unsigned int *>(static_cast<char *>(ws) +
                                                                              round_up(rows * S * c.dv * 4, 256) +
                                                                              round_up(rows * S * 4, 256));
    p.gaps = op.gaps_out;
    p.status = op.status_word;
    p.B = B; p.Hq = Hq; p.Lq = Lq; p.Lk = Lk; p.R = (int)R;
    p.nb = nb; p.num_splits = S; p.per_split = per_split; p.words = words;
    p.causal = causal ? 1 : 0;
    p.scale_log2 = (float)(scale * kLog2e);
    p.thr_log2 = log2_threshold(lambda);
    p.seed = op.seed_splits ? 1 : 0;
    e = launch_mla(p, tq, tk, calib, sm);
    if (e != cudaSuccess) return cuda_fail(e, "MLA split kernel");
    if (!calib) {
        CombineParams cp;
        cp.part_o = p.part_o;
        cp.part_lse = p.part_lse;
        cp.o = static_cast<uint16_t *>(o);
        cp.lse = lse;
        cp.rows = (int)rows;
        cp.num_splits = S;
        cp.dv = c.dv;
        cp.split_skips = p.split_skips;
        cp.n_counts = B * S;
        cp.skip_count = skip_count;
        e = launch_combine(cp, sm);
        if (e != cudaSuccess) return cuda_fail(e, "decode combine kernel");
    }
    if (own_ws) {
        e = cudaFreeAsync(ws, sm);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFreeAsync(workspace)");
    }
    return BLASST_OK;
}

// ------------------------------------------------------------------- decode
// A paged KV cache: pages [num_pages, Hkv, 64, d]; sequence b has seq_lens[b] keys in
// pages block_table[b * max_pages + i].  Both arrays are int32 in device memory.
struct PagedCache {
    const int *block_table;
    const int *seq_lens;
    int max_pages, num_pages;
};

// FP8 (e4m3) K/V cache: K = k_scale * e4m3, V = v_scale * e4m3.
struct Fp8Cache {
    float k_scale, v_scale;
};

blasst_status run_decode(const void *q, const void *k, const void *v, void *o, float *lse, int B, int Hq, int Hkv,
                         int Lq, int Lk, int d, float scale, float lambda, int causal, uint32_t *skip_mask,
                         unsigned long long *skip_count, void *stream, const blasst_opts *opts_in, bool calib,
                         const PagedCache *pg = nullptr, const Fp8Cache *f8 = nullptr) {
    blasst_opts op = read_opts(opts_in);
    Common c;
    blasst_status st = check_common(q, k, B, Hq, Hkv, Lq, Lk, d, scale, lambda, causal, op, &c);
    if (st != BLASST_OK) return st;
    if (!calib) {
        if (!v || !o || !lse) return BLASST_ERR_INVALID;
        if (!aligned(v, 16) || !aligned(o, 16) || !aligned(lse, 4)) return BLASST_ERR_INVALID;
    } else if (!op.gaps_out) {
        return BLASST_ERR_INVALID;
    }
    if (op.block_n != 0 && op.block_n != kDecodeBlockN) return BLASST_ERR_UNSUPPORTED;
    if (op.seed_splits && d != 128 && d != 576) return BLASST_ERR_UNSUPPORTED;  // split seeding: decode only
    if (pg && (d != 128 || c.dv != 128 || c.krs != d || c.vrs != c.dv)) return BLASST_ERR_UNSUPPORTED;
    if (f8) {
        if (!(std::isfinite(f8->k_scale) && f8->k_scale > 0.f && std::isfinite(f8->v_scale) && f8->v_scale > 0.f))
            return BLASST_ERR_INVALID;
        if (calib || pg || d != 128 || c.dv != 128 || c.krs != d || c.vrs != c.dv) return BLASST_ERR_UNSUPPORTED;
        if ((long long)(Hq / Hkv) * Lq > 16) return BLASST_ERR_UNSUPPORTED;  // tiles of up to 16 rows
    }
    if (d == 576) return run_mla(q, k, v, o, lse, B, Hq, Hkv, Lq, Lk, d, scale, lambda, causal, skip_mask, skip_count,
                                 stream, op, c, calib);
    if (d != 128 || c.dv != 128) return BLASST_ERR_UNSUPPORTED;
    const int G = Hq / Hkv;
    const long long R = (long long)G * Lq;
    // tiles of up to 16 rows: mma.sync kernel; 17..128 rows (MQA, large groups): tcgen05 kernel
    const bool wide = R > 16;
    if (R > 128) return BLASST_ERR_UNSUPPORTED;
    int S = 0;
    st = decode_split_count(d, op.num_splits, B, Hkv, (int)R, Lk, &S);
    if (st != BLASST_OK) return st;
    if (S > 65535) return BLASST_ERR_INVALID;
    if (wide && ((Lk + kDecodeBlockN - 1) / kDecodeBlockN + S - 1) / S > (op.seed_splits ? 1023 : 1024))
        return BLASST_ERR_UNSUPPORTED;  // wide tiles: at most 1024 ring entries per split (seed block included)
    if (Hkv > 65535 || B > 65535) return BLASST_ERR_UNSUPPORTED;
    if ((long long)S * Hkv * B > 0x7fffffffLL) return BLASST_ERR_UNSUPPORTED;  // one CTA (and count slot) per split
    const int nb = (Lk + kDecodeBlockN - 1) / kDecodeBlockN;
    const int per_split = (nb + S - 1) / S;
    if (per_split > kMaxBlocksPerSplit) return BLASST_ERR_UNSUPPORTED;

    cudaStream_t sm = reinterpret_cast<cudaStream_t>(stream);
    const int words = (nb + 31) / 32;
    const size_t rows = (size_t)B * Hq * Lq;
    const size_t need = blasst_decode_workspace_bytes(B, Hq, Lq, c.dv, S);

    void *ws = op.workspace;
    if (!calib && ws && op.workspace_bytes < need) return BLASST_ERR_WORKSPACE;

    // K/V: [planes, rows, d] with a plane per (sequence, KV head), or per (page, KV head)
    const long long planes = pg ? (long long)pg->num_pages * Hkv : (long long)B * Hkv;
    const long long plane_rows = pg ? kDecodeBlockN : Lk;
    CUtensorMap tk, tv;
    if (f8) {  // e4m3 rows of 128 bytes
        st = make_tmap_u8(&tk, k, plane_rows, planes, 64);
        if (st == BLASST_OK) st = make_tmap_u8(&tv, v, plane_rows, planes, 64);
        if (st != BLASST_OK) return st;
    } else {
        st = make_tmap(&tk, k, d, plane_rows, planes, c.krs, 64, 64);
        if (st != BLASST_OK) return st;
        if (!calib) {
            st = make_tmap(&tv, v, c.dv, plane_rows, planes, c.vrs, 64, 64);
            if (st != BLASST_OK) return st;
        } else {
            tv = tk;
        }
    }
    CUtensorMap tq;  // wide tiles: q as [B][Hq*Lq][128], 128-row boxes
    if (wide) {
        st = make_tmap(&tq, q, d, (long long)Hq * Lq, B, d, 64, 128);
        if (st != BLASST_OK) return st;
    }

    bool own_ws = false;
    if (!calib) {
        if (!ws) {
            cudaError_t e = cudaMallocAsync(&ws, need, sm);
            if (e != cudaSuccess) return cuda_fail(e, "cudaMallocAsync(workspace)");
            own_ws = true;
        }
    }
    cudaError_t e;
    if (skip_mask) {
        e = cudaMemsetAsync(skip_mask, 0, (size_t)B * Hkv * words * sizeof(uint32_t), sm);
        if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(skip_mask)");
    }
    // the calibration pass adds into skip_count; an attention call's split CTAs store their
    // counts in the workspace and the combine kernel writes the sum (no reset needed)
    if (skip_count && calib) {
        e = cudaMemsetAsync(skip_count, 0, sizeof(unsigned long long), sm);
        if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(skip_count)");
    }

    DecodeParams p;
    std::memset(&p, 0, sizeof p);
    p.q = static_cast<const uint16_t *>(q);
    p.part_o = calib ? nullptr : static_cast<float *>(ws);
    p.part_lse = calib ? nullptr : reinterpret_cast<float *>(static_cast<char *>(ws) + round_up(rows * S * c.dv * 4, 256));
    p.skip_mask = skip_mask;
    p.skip_count = calib ? skip_count : nullptr;
    p.split_skips = (calib || !skip_count) ? nullptr
                                           : reinterpret_cast<unsigned int *>(static_cast<char *>(ws) +
                                                                              round_up(rows * S * c.dv * 4, 256) +
                                                                              round_up(rows * S * 4, 256));
    p.gaps = op.gaps_out;
    p.status = op.status_word;
    p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.Lq = Lq; p.Lk = Lk; p.G = G; p.R = (int)R;
    p.nb = nb; p.num_splits = S; p.per_split = per_split; p.words = words;
    p.causal = causal ? 1 : 0;
    p.scale_log2 = (float)(scale * kLog2e * (f8 ? f8->k_scale : 1.f));
    p.thr_log2 = log2_threshold(lambda);
    p.seed = op.seed_splits ? 1 : 0;
    p.v_scale = f8 ? f8->v_scale : 1.f;
    if (pg) {
        p.block_table = pg->block_table;
        p.seq_lens = pg->seq_lens;
        p.num_pages = pg->num_pages;
    }
    if (f8) {
        e = launch_decode_fp8(p, tk, tv, R <= 8 ? 1 : 2, sm);
    } else if (wide) {
        e = launch_decode_wide(p, tq, tk, tv, calib, sm);
    } else {
        e = launch_decode(p, tk, tv, calib, R <= 8 ? 1 : 2, sm);
    }
    if (e != cudaSuccess) return cuda_fail(e, "decode split kernel");
    if (!calib) {
        CombineParams cp;
        cp.part_o = p.part_o;
        cp.part_lse = p.part_lse;
        cp.o = static_cast<uint16_t *>(o);
        cp.lse = lse;
        cp.rows = (int)rows;
        cp.num_splits = S;
        cp.dv = c.dv;
        cp.split_skips = p.split_skips;
        cp.n_counts = S * Hkv * B;
        cp.skip_count = skip_count;
        e = launch_combine(cp, sm);
        if (e != cudaSuccess) return cuda_fail(e, "decode combine kernel");
    }
    if (own_ws) {
        e = cudaFreeAsync(ws, sm);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFreeAsync(workspace)");
    }
    return BLASST_OK;
}

// ------------------------------------------------------------------ prefill
blasst_status run_prefill(const void *q, const void *k, const void *v, void *o, float *lse, int B, int Hq, int Hkv,
                          int Lq, int Lk, int d, float scale, float lambda, int causal, uint32_t *skip_mask,
                          unsigned long long *skip_count, void *stream, const blasst_opts *opts_in, bool calib,
                          bool novote = false) {
    blasst_opts op = read_opts(opts_in);
    Common c;
    blasst_status st = check_common(q, k, B, Hq, Hkv, Lq, Lk, d, scale, lambda, causal, op, &c);
    if (st != BLASST_OK) return st;
    if (op.seed_splits) return BLASST_ERR_UNSUPPORTED;  // prefill has no splits
    if (!calib) {
        if (!v || !o || !lse) return BLASST_ERR_INVALID;
        if (!aligned(v, 16) || !aligned(o, 16) || !aligned(lse, 4)) return BLASST_ERR_INVALID;
    } else if (!op.gaps_out) {
        return BLASST_ERR_INVALID;
    }
    if (op.block_n != 0 && op.block_n != kPrefillBlockN) return BLASST_ERR_UNSUPPORTED;
    if (d != 128 || c.dv != 128) return BLASST_ERR_UNSUPPORTED;
    if (B > 65535) return BLASST_ERR_UNSUPPORTED;
    const int nq = (Lq + kPrefillBlockM - 1) / kPrefillBlockM;
    const int nb = (Lk + kPrefillBlockN - 1) / kPrefillBlockN;
    const int words = (nb + 31) / 32;
    cudaStream_t sm = reinterpret_cast<cudaStream_t>(stream);

    CUtensorMap tq, tk, tv;
    st = make_tmap(&tq, q, d, Lq, (long long)B * Hq, d, 64, kPrefillBlockM);
    if (st != BLASST_OK) return st;
    st = make_tmap(&tk, k, d, Lk, (long long)B * Hkv, c.krs, 64, kPrefillBlockN);
    if (st != BLASST_OK) return st;
    if (!calib) {
        st = make_tmap(&tv, v, c.dv, Lk, (long long)B * Hkv, c.vrs, 64, kPrefillBlockN);
        if (st != BLASST_OK) return st;
    } else {
        tv = tk;
    }
    cudaError_t e;
    if (skip_count) {
        e = cudaMemsetAsync(skip_count, 0, sizeof(unsigned long long), sm);
        if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(skip_count)");
    }
    PrefillParams p;
    std::memset(&p, 0, sizeof p);
    p.o = static_cast<uint16_t *>(o);
    p.lse = lse;
    p.skip_mask = skip_mask;
    p.skip_count = skip_count;
    p.gaps = op.gaps_out;
    p.status = op.status_word;
    p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.Lq = Lq; p.Lk = Lk; p.G = Hq / Hkv;
    p.n_qtiles = nq; p.nb = nb; p.words = words;
    p.causal = causal ? 1 : 0;
    p.scale_log2 = (float)(scale * kLog2e);
    p.thr_log2 = log2_threshold(lambda);
    e = novote ? launch_prefill_novote(p, tq, tk, tv, sm) : launch_prefill(p, tq, tk, tv, calib, sm);
    if (e == cudaErrorNotSupported) return BLASST_ERR_UNSUPPORTED;
    if (e != cudaSuccess) return cuda_fail(e, "prefill kernel");
    return BLASST_OK;
}

size_t backward_ws_parts(int B, int Hq, int Lq, size_t *acc_bytes, size_t *row_bytes) {
    const size_t rows = (size_t)B * Hq * (size_t)(((long long)Lq + 127) / 128 * 128);
    *acc_bytes = round_up(rows * 128 * sizeof(float), 256);
    *row_bytes = round_up(rows * sizeof(float), 256);
    return *acc_bytes + 2 * *row_bytes;
}

blasst_status run_backward(const void *q, const void *k, const void *v, const void *o, const float *lse,
                           const void *dout, void *dq, void *dk, void *dv, int B, int Hq, int Hkv, int Lq, int Lk,
                           int d, float scale, int causal, const uint32_t *skip_mask, void *stream,
                           const blasst_opts *opts_in) {
    blasst_opts op = read_opts(opts_in);
    Common c;
    blasst_status st = check_common(q, k, B, Hq, Hkv, Lq, Lk, d, scale, 0.f, causal, op, &c);
    if (st != BLASST_OK) return st;
    if (!v || !o || !lse || !dout || !dq || !dk || !dv) return BLASST_ERR_INVALID;
    if (!aligned(v, 16) || !aligned(o, 16) || !aligned(dout, 16) || !aligned(dq, 16) || !aligned(dk, 16) ||
        !aligned(dv, 16) || !aligned(lse, 4) || (skip_mask && !aligned(skip_mask, 4)))
        return BLASST_ERR_INVALID;
    if (op.seed_splits || op.mode) return BLASST_ERR_UNSUPPORTED;
    if (op.block_n != 0 && op.block_n != kPrefillBlockN) return BLASST_ERR_UNSUPPORTED;
    if (d != 128 || c.dv != 128 || c.krs != 128 || c.vrs != 128) return BLASST_ERR_UNSUPPORTED;
    if (B > 65535) return BLASST_ERR_UNSUPPORTED;
    const int nq = (Lq + kPrefillBlockM - 1) / kPrefillBlockM;
    const int nb = (Lk + kPrefillBlockN - 1) / kPrefillBlockN;
    if ((long long)nb * Hkv > 0x7fffffffLL) return BLASST_ERR_UNSUPPORTED;
    size_t acc_bytes, row_bytes;
    const size_t need = backward_ws_parts(B, Hq, Lq, &acc_bytes, &row_bytes);
    void *ws = op.workspace;
    if (ws && op.workspace_bytes < need) return BLASST_ERR_WORKSPACE;
    cudaStream_t sm = reinterpret_cast<cudaStream_t>(stream);

    CUtensorMap tq, tdo, tk, tv;
    st = make_tmap(&tq, q, d, Lq, (long long)B * Hq, d, 64, kPrefillBlockM);
    if (st != BLASST_OK) return st;
    st = make_tmap(&tdo, dout, d, Lq, (long long)B * Hq, d, 64, kPrefillBlockM);
    if (st != BLASST_OK) return st;
    st = make_tmap(&tk, k, d, Lk, (long long)B * Hkv, d, 64, kPrefillBlockN);
    if (st != BLASST_OK) return st;
    st = make_tmap(&tv, v, d, Lk, (long long)B * Hkv, d, 64, kPrefillBlockN);
    if (st != BLASST_OK) return st;
    const bool own_ws = (ws == nullptr);
    cudaError_t e;
    if (own_ws) {
        e = cudaMallocAsync(&ws, need, sm);
        if (e != cudaSuccess) return cuda_fail(e, "cudaMallocAsync(workspace)");
    }
    uint8_t *w8 = static_cast<uint8_t *>(ws);
    BwdParams p;
    std::memset(&p, 0, sizeof p);
    p.o = static_cast<const uint16_t *>(o);
    p.dout = static_cast<const uint16_t *>(dout);
    p.lse = lse;
    p.dq_acc = reinterpret_cast<float *>(w8);
    p.neg_lse2 = reinterpret_cast<float *>(w8 + acc_bytes);
    p.neg_sdelta = reinterpret_cast<float *>(w8 + acc_bytes + row_bytes);
    p.dq = static_cast<uint16_t *>(dq);
    p.dk = static_cast<uint16_t *>(dk);
    p.dv = static_cast<uint16_t *>(dv);
    p.skip_mask = skip_mask;
    p.status = op.status_word;
    p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.Lq = Lq; p.Lk = Lk; p.G = Hq / Hkv;
    p.Lq_pad = nq * kPrefillBlockM; p.nq = nq; p.nb = nb; p.words = (nb + 31) / 32;
    p.causal = causal ? 1 : 0;
    p.scale_log2 = (float)(scale * kLog2e);
    p.scale = scale;
    e = launch_backward(p, tq, tdo, tk, tv, sm);
    blasst_status rs = BLASST_OK;
    if (e != cudaSuccess) rs = cuda_fail(e, "backward kernels");
    if (own_ws) {
        cudaError_t e2 = cudaFreeAsync(ws, sm);
        if (e2 != cudaSuccess && rs == BLASST_OK) rs = cuda_fail(e2, "cudaFreeAsync(workspace)");
    }
    return rs;
}

}  // namespace

extern "C" {

blasst_status blasst_prefill_backward(const void *q, const void *k, const void *v, const void *o, const float *lse,
                                      const void *dout, void *dq, void *dk, void *dv, int B, int Hq, int Hkv,
                                      int Lq, int Lk, int d, float scale, int causal, const uint32_t *skip_mask,
                                      void *stream, const blasst_opts *opts) {
    return run_backward(q, k, v, o, lse, dout, dq, dk, dv, B, Hq, Hkv, Lq, Lk, d, scale, causal, skip_mask, stream,
                        opts);
}

size_t blasst_backward_workspace_bytes(int B, int Hq, int Lq) {
    if (B <= 0 || Hq <= 0 || Lq <= 0) return 0;
    size_t a, r;
    return backward_ws_parts(B, Hq, Lq, &a, &r);
}

blasst_status blasst_prefill(const void *q, const void *k, const void *v, void *o, float *lse, int B, int Hq, int Hkv,
                             int Lq, int Lk, int d, float scale, float lambda, int causal, uint32_t *skip_mask,
                             unsigned long long *skip_count, void *stream, const blasst_opts *opts) {
    return run_prefill(q, k, v, o, lse, B, Hq, Hkv, Lq, Lk, d, scale, lambda, causal, skip_mask, skip_count, stream,
                       opts, false);
}

blasst_status blasst_measure_prefill_novote(const void *q, const void *k, const void *v, void *o, float *lse, int B,
                                            int Hq, int Hkv, int Lq, int Lk, int d, float scale, float lambda,
                                            int causal, uint32_t *skip_mask, unsigned long long *skip_count,
                                            void *stream, const blasst_opts *opts) {
    return run_prefill(q, k, v, o, lse, B, Hq, Hkv, Lq, Lk, d, scale, lambda, causal, skip_mask, skip_count, stream,
                       opts, false, true);
}

blasst_status blasst_decode(const void *q, const void *k, const void *v, void *o, float *lse, int B, int Hq, int Hkv,
                            int Lq, int Lk, int d, float scale, float lambda, int causal, uint32_t *skip_mask,
                            unsigned long long *skip_count, void *stream, const blasst_opts *opts) {
    return run_decode(q, k, v, o, lse, B, Hq, Hkv, Lq, Lk, d, scale, lambda, causal, skip_mask, skip_count, stream,
                      opts, false);
}

blasst_status blasst_decode_fp8(const void *q, const void *k8, const void *v8, void *o, float *lse, int B, int Hq,
                               int Hkv, int Lq, int Lk, int d, float scale, float k_scale, float v_scale,
                               float lambda, int causal, uint32_t *skip_mask, unsigned long long *skip_count,
                               void *stream, const blasst_opts *opts) {
    if (!v8) return BLASST_ERR_INVALID;
    const Fp8Cache f8{k_scale, v_scale};
    return run_decode(q, k8, v8, o, lse, B, Hq, Hkv, Lq, Lk, d, scale, lambda, causal, skip_mask, skip_count, stream,
                      opts, false, nullptr, &f8);
}

blasst_status blasst_decode_paged(const void *q, const void *k_pages, const void *v_pages, void *o,
                                 float *lse, const int *block_table, const int *seq_lens, int B, int Hq,
                                             int Hkv, int Lq, int max_pages, int num_pages, int d, float scale,
                                             float lambda, int causal, uint32_t *skip_mask,
                                             unsigned long long *skip_count, void *stream, const blasst_opts *opts) {
    if (!block_table || !seq_lens || !aligned(block_table, 4) || !aligned(seq_lens, 4)) return BLASST_ERR_INVALID;
    if (max_pages <= 0 || num_pages <= 0) return BLASST_ERR_INVALID;
    if ((long long)max_pages * kDecodeBlockN > INT_MAX || (long long)num_pages * (Hkv > 0 ? Hkv : 1) > INT_MAX)
        return BLASST_ERR_INVALID;
    const PagedCache pg{block_table, seq_lens, max_pages, num_pages};
    return run_decode(q, k_pages, v_pages, o, lse, B, Hq, Hkv, Lq, max_pages * kDecodeBlockN, d, scale, lambda,
                      causal, skip_mask, skip_count, stream, opts, false, &pg);
}

blasst_status blasst_calibrate(const void *q, const void *k, const void *v, void *o, float *lse, int B, int Hq,
                               int Hkv, int Lq, int Lk, int d, float scale, float lambda, int causal,
                               uint32_t *skip_mask, unsigned long long *skip_count, void *stream,
                               const blasst_opts *opts) {
    (void)v;
    (void)o;
    (void)lse;
    blasst_opts op = read_opts(opts);
    if (op.mode == 1)
        return run_decode(q, k, nullptr, nullptr, nullptr, B, Hq, Hkv, Lq, Lk, d, scale, lambda, causal, skip_mask,
                          skip_count, stream, opts, true);
    if (op.mode != 0) return BLASST_ERR_INVALID;
    return run_prefill(q, k, nullptr, nullptr, nullptr, B, Hq, Hkv, Lq, Lk, d, scale, lambda, causal, skip_mask,
                       skip_count, stream, opts, true);
}

blasst_status blasst_calibrate_fit(const double *L, const double *lambda, const double *sparsity, int n,
                                   double *alpha, double *beta) {
    if (!L || !lambda || !sparsity || !alpha || !beta || n < 2) return BLASST_ERR_INVALID;
    double sx = 0, sy = 0, sxx = 0, sxy = 0;
    for (int i = 0; i < n; i++) {
        if (!(L[i] > 0) || !(lambda[i] > 0) || !std::isfinite(sparsity[i])) return BLASST_ERR_INVALID;
        const double x = sparsity[i], y = std::log(lambda[i] * L[i]);
        sx += x;
        sy += y;
        sxx += x * x;
        sxy += x * y;
    }
    const double den = n * sxx - sx * sx;
    if (den == 0.0) return BLASST_ERR_INVALID;
    *beta = (n * sxy - sx * sy) / den;
    *alpha = std::exp((sy - *beta * sx) / n);
    return BLASST_OK;
}

blasst_status blasst_calibrate_threshold(const float *gaps, long long n, double target, double *lambda_out,
                                         double *achieved_out) {
    if (!gaps || n < 0 || !lambda_out || !(target >= 0.0 && target <= 1.0)) return BLASST_ERR_INVALID;
    long long n_vis = 0;
    std::vector<double> cand;
    for (long long i = 0; i < n; i++) {
        const float g = gaps[i];
        if (std::isnan(g)) continue;
        n_vis++;
        if (std::isfinite(g) && g < 0.f) cand.push_back((double)g);
    }
    std::sort(cand.begin(), cand.end());
    long long want = n_vis ? (long long)std::llround(target * (double)n_vis) : 0;
    want = std::max(0LL, std::min<long long>(want, (long long)cand.size()));
    double lam = 0.0;
    long long got = 0;
    if (want > 0) {
        const double lo = cand[want - 1];
        const double hi = want < (long long)cand.size() ? cand[want] : 0.0;
        double ln_lam = hi > lo ? 0.5 * (lo + hi) : std::nextafter(lo, INFINITY);
        lam = std::min(std::exp(ln_lam), std::nextafter(1.0, 0.0));
        // what the device decides: gap (log2 units, fp32) < log2(lambda) (fp32)
        const float thr = log2_threshold((float)lam);
        for (double g : cand)
            if ((float)((float)g * (float)kLog2e) < thr) got++;
    }
    *lambda_out = lam;
    if (achieved_out) *achieved_out = n_vis ? (double)got / (double)n_vis : 0.0;
    return BLASST_OK;
}

int blasst_decode_pick_splits(int B, int Hkv, int Lk, int num_sms) {
    if (B <= 0 || Hkv <= 0 || Lk <= 0 || num_sms <= 0) return 1;
    const long long groups = (long long)B * Hkv;
    const long long nb = (Lk + kDecodeBlockN - 1) / kDecodeBlockN;
    const long long cap = std::max(1LL, std::min(64LL, nb / 32));  // at least 32 blocks per split
    const long long want = (16LL * num_sms + groups - 1) / groups;  // about 16 CTAs per SM over the call
    return (int)std::max(1LL, std::min(cap, want));
}

int blasst_decode_pick_splits_rows(int B, int Hkv, int rows, int Lk, int num_sms) {
    if (rows <= 16) return blasst_decode_pick_splits(B, Hkv, Lk, num_sms);
    if (B <= 0 || Hkv <= 0 || Lk <= 0 || num_sms <= 0) return 1;
    // wide tiles (tcgen05 kernel, two CTAs per SM): as many splits as keep the grid within two
    // full waves of two CTAs per SM, under the same cap
    const long long groups = (long long)B * Hkv;
    const long long nb = (Lk + kDecodeBlockN - 1) / kDecodeBlockN;
    const long long cap = std::max(1LL, std::min(64LL, nb / 32));
    const long long want = 4LL * num_sms / groups;
    return (int)std::max(1LL, std::min(cap, want));
}

size_t blasst_decode_workspace_bytes(int B, int Hq, int Lq, int dv, int num_splits) {
    if (B <= 0 || Hq <= 0 || Lq <= 0 || dv < 0 || num_splits < 0) return 0;
    const size_t S = num_splits ? num_splits : 16;
    const size_t rows = (size_t)B * Hq * Lq;
    const size_t dvv = dv ? dv : 128;
    // partial O, partial lse, then one skip-count slot per split CTA (at most B * Hq * S)
    return round_up(rows * S * dvv * 4, 256) + round_up(rows * S * 4, 256) + round_up((size_t)B * Hq * S * 4, 256);
}

long long blasst_visited_pairs(int B, int Hq, int Hkv, int Lq, int Lk, int causal, int is_decode,
                               const blasst_opts *opts) {
    blasst_opts op = read_opts(opts);
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Lq <= 0 || Lk <= 0 || Hq % Hkv) return -1;
    if (causal && Lq > Lk) return -1;
    if (is_decode) {
        const int bn = op.block_n ? op.block_n : kDecodeBlockN;
        const long long nb = (Lk + bn - 1) / bn;
        // every key block is seen by the last query of the tile
        return (long long)B * Hkv * nb;
    }
    const int bn = op.block_n ? op.block_n : kPrefillBlockN;
    const long long nb = (Lk + bn - 1) / bn;
    const int nq = (Lq + kPrefillBlockM - 1) / kPrefillBlockM;
    long long per_head = 0;
    for (int t = 0; t < nq; t++) {
        if (!causal) {
            per_head += nb;
        } else {
            const long long last_row = std::min<long long>(Lq, (long long)(t + 1) * kPrefillBlockM) - 1;
            const long long last_key = last_row + (Lk - Lq);
            per_head += std::min<long long>(nb, last_key / bn + 1);
        }
    }
    return per_head * B * Hq;
}

const char *blasst_status_string(blasst_status s) {
    switch (s) {
        case BLASST_OK: return "ok";
        case BLASST_ERR_INVALID: return "invalid argument";
        case BLASST_ERR_UNSUPPORTED: return "unsupported configuration";
        case BLASST_ERR_WORKSPACE: return "workspace too small";
        case BLASST_ERR_CUDA: return "CUDA error";
        case BLASST_ERR_TIMEOUT: return "device wait timed out";
    }
    return "unknown status";
}

const char *blasst_last_error(void) { return g_last_error; }

}  // extern "C"
