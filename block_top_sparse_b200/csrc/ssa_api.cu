// ssa_api.cu -- the C ABI of libssa (declared in include/ssa.h): argument
// validation, workspace carving, TMA descriptor set-up and kernel launches.
// All kernels are compiled into this one translation unit.

#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>

#include "ssa.h"

#include "device.cuh"
#include "pool_select.cuh"
#include "aux_kernels.cuh"
#include "attn_simt.cuh"
#include "attn_tc.cuh"
#include "attn_bwd.cuh"
#include "decode.cuh"
#include "rope.cuh"

using namespace ssa;

namespace {

struct Shape {
    int B, H, T, d, s, k, dtype;
    float scale;
    int Hk, G;         // key/value heads, query heads per key/value head
    size_t BH, rows;   // query heads B*H, query rows B*H*T
    size_t BHk, krows; // key/value heads B*Hk, key rows B*Hk*T
    int nb;
    size_t esz;       // element size in bytes
    bool tc;          // tensor-core path (bf16, d == 128)
};

ssa_status_t check_dims(const ssa_dims_t *dims, Shape &S, bool need_k) {
    if (!dims) return SSA_ERR_INVALID_ARG;
    S.B = dims->B;
    S.H = dims->H;
    S.T = dims->T;
    S.d = dims->d;
    S.s = dims->s;
    S.k = dims->k;
    S.dtype = dims->dtype;
    S.scale = dims->scale;
    if (S.B < 1 || S.H < 1 || S.T < 1 || S.d < 1 || S.s < 1) return SSA_ERR_INVALID_ARG;
    if (S.dtype != SSA_DT_BF16 && S.dtype != SSA_DT_FP32) return SSA_ERR_INVALID_ARG;
    if (!(std::isfinite(S.scale) && S.scale > 0.f)) return SSA_ERR_INVALID_ARG;
    if (S.d != 64 && S.d != 128) return SSA_ERR_UNSUPPORTED;
    if (S.s != 64 && S.s != 128) return SSA_ERR_UNSUPPORTED;
    if (S.T % S.s != 0) return SSA_ERR_UNSUPPORTED;
    S.Hk = dims->Hkv ? dims->Hkv : S.H;
    if (S.Hk < 1 || S.H % S.Hk != 0) return SSA_ERR_INVALID_ARG;
    S.G = S.H / S.Hk;
    S.BH = static_cast<size_t>(S.B) * S.H;
    S.rows = S.BH * S.T;
    S.BHk = static_cast<size_t>(S.B) * S.Hk;
    S.krows = S.BHk * S.T;
    if (S.rows > 0x7FFFFFFFull) return SSA_ERR_UNSUPPORTED;  // TMA row coordinates are int32
    S.nb = S.T / S.s;
    if (need_k) {
        if (S.k < 1 || S.k > S.nb) return SSA_ERR_INVALID_ARG;
        if (static_cast<int64_t>(S.T) * S.k > 0x7FFFFFFFll) return SSA_ERR_UNSUPPORTED;
    }
    S.esz = S.dtype == SSA_DT_BF16 ? 2 : 4;
    S.tc = S.dtype == SSA_DT_BF16 && S.d == 128;
    // a tensor-core tile holds 128 / G list entries for each of the G heads of a group
    if (S.tc && 128 % S.G != 0) return SSA_ERR_UNSUPPORTED;
    // the sparse index packs (t << 8) | slot into an int32
    if (need_k && S.tc && (S.k > 256 || S.T >= (1 << 23))) return SSA_ERR_UNSUPPORTED;
    // list positions of the whole index (and TMA row coordinates of the G partial rows per entry) fit an int32
    if (need_k && S.tc && S.BHk * list_stride(S.T, S.k, S.nb) * S.G >= (size_t(1) << 31)) return SSA_ERR_UNSUPPORTED;
    // one warp's staging of the index fill must fit in shared memory
    if (need_k && S.tc && index_fill_warp_ints(S.nb, S.k) * 4 > 227 * 1024) return SSA_ERR_UNSUPPORTED;
    return SSA_OK;
}

inline size_t align_up(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Layout of the inverse selection index (the `index` buffer of ssa_sparse_index, or
// the head of a sparse call's workspace when the caller passes none).
struct IndexWs {
    int *cnt, *lstart, *llen;
    int32_t *entries;  // per head: list_stride(T, k, nb) entries, block lists on 128-entry boundaries
    int32_t *pos;      // [B*H*T, k] list position of every (query, slot), -1 when unused
    int32_t *order;    // [B*Hk*nb] launch order of the (head, block) units, heaviest first
    int nch;
};

size_t index_bytes(const Shape &S) {
    if (!S.tc) return 0;
    const size_t nch = (S.T + kIdxChunk - 1) / kIdxChunk;
    return align_up(S.BHk * nch * S.nb * 4) + 3 * align_up(S.BHk * S.nb * 4) +
           align_up(S.BHk * list_stride(S.T, S.k, S.nb) * 4) + align_up(S.krows * S.k * 4);
}

IndexWs carve_index(const Shape &S, const void *base) {
    IndexWs W;
    uint8_t *p = static_cast<uint8_t *>(const_cast<void *>(base));
    W.nch = (S.T + kIdxChunk - 1) / kIdxChunk;
    W.cnt = reinterpret_cast<int *>(p);
    p += align_up(S.BHk * W.nch * S.nb * 4);
    W.lstart = reinterpret_cast<int *>(p);
    p += align_up(S.BHk * S.nb * 4);
    W.llen = reinterpret_cast<int *>(p);
    p += align_up(S.BHk * S.nb * 4);
    W.entries = reinterpret_cast<int32_t *>(p);
    p += align_up(S.BHk * list_stride(S.T, S.k, S.nb) * 4);
    W.pos = reinterpret_cast<int32_t *>(p);
    p += align_up(S.krows * S.k * 4);
    W.order = reinterpret_cast<int32_t *>(p);
    return W;
}

size_t ws_bytes_for(const Shape &S, int op) {
    switch (op) {
        case SSA_OP_SPARSE_INDEX:
            return index_bytes(S);
        case SSA_OP_SPARSE_FWD:
            if (!S.tc) return 0;
            // index (used when the caller passes none) | fp16 partial outputs and fp32 partial lse,
            // G rows per list position | range exponent of every key block, then a flag word
            return index_bytes(S) + align_up(S.BHk * list_stride(S.T, S.k, S.nb) * S.G * (128 * 2 + 4)) +
                   align_up(S.BHk * S.nb * 4 + 4);
        case SSA_OP_SPARSE_BWD:
            // D | index (used when the caller passes none) | fp32 dQ accumulator
            if (S.tc) return align_up(S.rows * 4) + index_bytes(S) + align_up(S.rows * S.d * 4);
            [[fallthrough]];
        case SSA_OP_FULL_BWD: {
            size_t b = align_up(S.rows * 4) + align_up(S.rows * S.d * 4);  // D, dQacc
            if (!S.tc) b += 2 * align_up(S.krows * S.d * 4);               // dKacc, dVacc
            return b;
        }
        case SSA_OP_FULL_FWD:
            return 0;
        case SSA_OP_ALIGN_FWD:
            return align_up(kAlignBlocks * 4);
        case SSA_OP_DECODE:
            // per (sequence, query head, slot): fp32 partial output and log-sum-exp
            return align_up(S.BH * S.k * S.d * 4) + align_up(S.BH * S.k * 4);
        default:
            return 0;
    }
}

ssa_status_t check_ws(const Shape &S, int op, const void *ws, size_t ws_bytes) {
    const size_t need = ws_bytes_for(S, op);
    if (need == 0) return SSA_OK;
    if (!ws || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 15u)) return SSA_ERR_WORKSPACE;
    return SSA_OK;
}

// Bits of a backward call's `accumulate`; fp32 gradients are written with 16-byte accesses and
// reduced into by the TMA unit, so their base addresses must be 16-byte aligned.
ssa_status_t check_grads(int accumulate, const void *dQ, const void *dK, const void *dV) {
    if (accumulate & ~static_cast<int>(SSA_BWD_ACCUMULATE | SSA_BWD_GRAD_FP32)) return SSA_ERR_INVALID_ARG;
    if ((accumulate & SSA_BWD_GRAD_FP32) &&
        ((reinterpret_cast<uintptr_t>(dQ) | reinterpret_cast<uintptr_t>(dK) | reinterpret_cast<uintptr_t>(dV)) & 15u))
        return SSA_ERR_INVALID_ARG;
    return SSA_OK;
}

ssa_status_t launch_status() {
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? SSA_OK : SSA_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// TMA descriptors: 2D view [rows, 128] of a bf16 tensor, box 64 columns x box_rows.
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

bool make_tmap(CUtensorMap *m, const void *base, size_t rows, int box_rows) {
    EncodeTiledFn f = encode_fn();
    if (!f) return false;
    const cuuint64_t gdim[2] = {128, rows};
    const cuuint64_t gstride[1] = {128 * 2};
    const cuuint32_t box[2] = {64, static_cast<cuuint32_t>(box_rows)};
    const cuuint32_t estride[2] = {1, 1};
    return f(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), gdim, gstride, box, estride,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// fp32 view [rows, 128] of the dQ accumulator, box 32 columns x 128 rows (128-byte rows, swizzled).
bool make_tmap_f32(CUtensorMap *m, const void *base, size_t rows) {
    EncodeTiledFn f = encode_fn();
    if (!f) return false;
    const cuuint64_t gdim[2] = {128, rows};
    const cuuint64_t gstride[1] = {128 * 4};
    const cuuint32_t box[2] = {32, 128};
    const cuuint32_t estride[2] = {1, 1};
    return f(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void *>(base), gdim, gstride, box, estride,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <typename K>
bool set_smem(K kernel, size_t bytes) {
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes)) ==
           cudaSuccess;
}

unsigned grid_for(size_t n, unsigned per_block) {
    size_t g = (n + per_block - 1) / per_block;
    if (g > 148u * 32u) g = 148u * 32u;
    return static_cast<unsigned>(g ? g : 1);
}

template <typename T, int KPL>
ssa_status_t launch_select(const Shape &S, const void *Q, const float *Kbar, int32_t *idx, size_t sm, cudaStream_t st) {
    if (!set_smem(select_kernel<T, KPL>, sm)) return SSA_ERR_CUDA;
    select_kernel<T, KPL><<<dim3(S.T / kSelQ, S.BHk), 256, sm, st>>>((const T *)Q, Kbar, idx, S.T, S.d, S.s, S.k, S.nb,
                                                                      S.G);
    return SSA_OK;
}

// Inverse selection index: entries of block j of head bh (query order) and the list
// position of every (query, slot).
ssa_status_t build_index(const Shape &S, const int32_t *idx, const IndexWs &W, cudaStream_t st) {
    const size_t hbytes = static_cast<size_t>(S.nb) * 4;
    if (!set_smem(index_count_kernel, hbytes)) return SSA_ERR_CUDA;
    index_count_kernel<<<dim3(W.nch, S.BHk), 256, hbytes, st>>>(idx, W.cnt, S.T, S.k, S.nb, W.nch);
    index_scan_kernel<<<S.BHk, 1024, 0, st>>>(W.cnt, W.lstart, W.llen, S.nb, W.nch);
    // four warps (chunks) per CTA while their staging fits comfortably, else one
    const size_t wbytes = index_fill_warp_ints(S.nb, S.k) * 4;
    const int wpc = wbytes * 4 <= 160 * 1024 ? 4 : 1;
    if (!set_smem(index_fill_kernel, wbytes * wpc)) return SSA_ERR_CUDA;
    index_fill_kernel<<<dim3((W.nch + wpc - 1) / wpc, S.BHk), 32 * wpc, wbytes * wpc, st>>>(
        idx, W.cnt, W.entries, W.pos, S.T, S.k, S.nb, W.nch);
    unit_order_kernel<<<1, 1024, 0, st>>>(W.llen, W.order, static_cast<int>(S.BHk) * S.nb, kTileQ / S.G);
    return launch_status();
}

template <typename T>
void launch_simt_fwd(const Shape &S, const void *Q, const void *K, const void *V, const int32_t *idx, void *O,
                     void *O_lo, float *lse, cudaStream_t st) {
    const unsigned g = static_cast<unsigned>((S.rows + 7) / 8);
    T *lo = sizeof(T) == 2 ? (T *)O_lo : nullptr;  // the residual is only kept for bf16 outputs
    if (S.d == 64)
        simt_fwd_kernel<T, 2><<<g, 256, 0, st>>>((const T *)Q, (const T *)K, (const T *)V, idx, (T *)O, lo, lse,
                                                 S.rows, S.T, S.s, S.k, S.scale, S.G);
    else
        simt_fwd_kernel<T, 4><<<g, 256, 0, st>>>((const T *)Q, (const T *)K, (const T *)V, idx, (T *)O, lo, lse,
                                                 S.rows, S.T, S.s, S.k, S.scale, S.G);
}

template <typename T>
ssa_status_t simt_bwd(const Shape &S, const void *Q, const void *K, const void *V, const void *O, const void *O_lo,
                      const float *lse, const void *dO, const int32_t *idx, void *dQ, void *dK, void *dV,
                      int accumulate, void *ws, cudaStream_t st) {
    uint8_t *p = static_cast<uint8_t *>(ws);
    float *Dvec = reinterpret_cast<float *>(p);
    p += align_up(S.rows * 4);
    float *dQacc = reinterpret_cast<float *>(p);
    p += align_up(S.rows * S.d * 4);
    float *dKacc = reinterpret_cast<float *>(p);
    p += align_up(S.krows * S.d * 4);
    float *dVacc = reinterpret_cast<float *>(p);
    const size_t n = S.rows * S.d, nk = S.krows * S.d;
    if (cudaMemsetAsync(dKacc, 0, nk * 4, st) != cudaSuccess || cudaMemsetAsync(dVacc, 0, nk * 4, st) != cudaSuccess)
        return SSA_ERR_CUDA;
    const unsigned g = static_cast<unsigned>((S.rows + 7) / 8);
    bwd_prep_kernel<T><<<g, 256, 0, st>>>((const T *)dO, (const T *)O, sizeof(T) == 2 ? (const T *)O_lo : nullptr,
                                          Dvec, dQacc, S.rows, S.d);
    if (S.d == 64)
        simt_bwd_kernel<T, 2><<<g, 256, 0, st>>>((const T *)Q, (const T *)K, (const T *)V, (const T *)dO, idx, lse,
                                                 Dvec, dQacc, dKacc, dVacc, S.rows, S.T, S.s, S.k, S.scale, S.G);
    else
        simt_bwd_kernel<T, 4><<<g, 256, 0, st>>>((const T *)Q, (const T *)K, (const T *)V, (const T *)dO, idx, lse,
                                                 Dvec, dQacc, dKacc, dVacc, S.rows, S.T, S.s, S.k, S.scale, S.G);
    const unsigned ge = grid_for(n, 256), gk = grid_for(nk, 256);
    const int acc = accumulate & SSA_BWD_ACCUMULATE;
    if ((accumulate & SSA_BWD_GRAD_FP32) || sizeof(T) == 4) {
        acc_to_out_kernel<float><<<ge, 256, 0, st>>>(dQacc, (float *)dQ, n, acc);
        acc_to_out_kernel<float><<<gk, 256, 0, st>>>(dKacc, (float *)dK, nk, acc);
        acc_to_out_kernel<float><<<gk, 256, 0, st>>>(dVacc, (float *)dV, nk, acc);
    } else {
        acc_to_out_kernel<T><<<ge, 256, 0, st>>>(dQacc, (T *)dQ, n, acc);
        acc_to_out_kernel<T><<<gk, 256, 0, st>>>(dKacc, (T *)dK, nk, acc);
        acc_to_out_kernel<T><<<gk, 256, 0, st>>>(dVacc, (T *)dV, nk, acc);
    }
    return launch_status();
}

// Tensor-core backward shared by both streams.
ssa_status_t tc_bwd(const Shape &S, const void *Q, const void *K, const void *V, const void *O, const void *O_lo,
                    const float *lse, const void *dO, const int32_t *idx, const void *index, void *dQ, void *dK,
                    void *dV, int accumulate, void *ws, cudaStream_t st) {
    uint8_t *p = static_cast<uint8_t *>(ws);
    float *Dvec = reinterpret_cast<float *>(p);
    p += align_up(S.rows * 4);
    const bool sparse = idx != nullptr;
    IndexWs W{};
    if (sparse) {
        // the caller's index, or one built here in the workspace
        W = carve_index(S, index ? index : p);
        p += index_bytes(S);
        if (!index) {
            const ssa_status_t e = build_index(S, idx, W, st);
            if (e != SSA_OK) return e;
        }
    }
    // fp32 dQ accumulator: TMA reduce-adds of whole tiles (full) or vector reductions of gathered
    // rows (sparse); zeroed by the prep kernel, converted (and added to dQ when accumulating) after.
    // With fp32 gradients the caller's dQ is the accumulator itself (zeroed unless accumulating).
    const bool acc = (accumulate & SSA_BWD_ACCUMULATE) != 0, g32 = (accumulate & SSA_BWD_GRAD_FP32) != 0;
    float *dQacc = g32 ? static_cast<float *>(dQ) : reinterpret_cast<float *>(p);
    float *zero_acc = (g32 && acc) ? nullptr : dQacc;
    if (((reinterpret_cast<uintptr_t>(O) | reinterpret_cast<uintptr_t>(O_lo)) & 7u) == 0) {  // 8-byte row loads
        const unsigned g = static_cast<unsigned>((S.rows + 8 * kPrepRows - 1) / (8 * kPrepRows));
        bwd_prep_bf16_kernel<<<g, 256, 0, st>>>((const __nv_bfloat16 *)dO, (const __nv_bfloat16 *)O,
                                                (const __nv_bfloat16 *)O_lo, Dvec, zero_acc, S.rows);
    } else {
        const unsigned g = static_cast<unsigned>((S.rows + 7) / 8);
        bwd_prep_kernel<__nv_bfloat16><<<g, 256, 0, st>>>((const __nv_bfloat16 *)dO, (const __nv_bfloat16 *)O,
                                                           (const __nv_bfloat16 *)O_lo, Dvec, zero_acc, S.rows, S.d);
    }
    const int nkv = sparse ? S.s : 128;
    CUtensorMap tmK, tmV, tmQ, tmdO, tmdQ;
    if (!make_tmap(&tmK, K, S.krows, nkv) || !make_tmap(&tmV, V, S.krows, nkv) || !make_tmap(&tmQ, Q, S.rows, 128) ||
        !make_tmap(&tmdO, dO, S.rows, 128) || !make_tmap_f32(&tmdQ, dQacc, S.rows))
        return SSA_ERR_CUDA;
    BwdArgs a{};
    a.Q = (const __nv_bfloat16 *)Q;
    a.dO = (const __nv_bfloat16 *)dO;
    a.lse = lse;
    a.Dvec = Dvec;
    a.dQacc = dQacc;
    a.dK = dK;
    a.dV = dV;
    a.entries = W.entries;
    a.lstart = W.lstart;
    a.llen = W.llen;
    a.order = sparse ? W.order : nullptr;
    a.BH = static_cast<int>(S.BHk);
    a.G = S.G;
    a.T = S.T;
    a.k = S.k;
    a.nb = S.nb;
    a.sparse = sparse ? 1 : 0;
    a.accumulate = acc ? 1 : 0;
    a.grad_fp32 = g32 ? 1 : 0;
    a.scale = S.scale;
    a.scale_log2 = S.scale * kLog2e;
    const unsigned units = static_cast<unsigned>(S.BHk * (sparse ? S.nb : (S.T + 127) / 128));
    const bool gq = S.G > 1;
    // the grouped-head instantiations carry the group arithmetic; one query head per key head does not
    auto run = [&](auto kernel, size_t sm) {
        if (!set_smem(kernel, sm)) return false;
        kernel<<<units, kBwdThreads, sm, st>>>(tmK, tmV, tmQ, tmdO, tmdQ, a);
        return true;
    };
    const size_t sm128 = BwdSmem<128>::kTotal + 1024, sm64 = BwdSmem<64>::kTotal + 1024;
    const bool launched = nkv == 128 ? (gq ? run(attn_bwd_kernel<128, true>, sm128) : run(attn_bwd_kernel<128, false>, sm128))
                                     : (gq ? run(attn_bwd_kernel<64, true>, sm64) : run(attn_bwd_kernel<64, false>, sm64));
    if (!launched) return SSA_ERR_CUDA;
    if (!g32) {
        const size_t n = S.rows * S.d;
        acc_to_out_kernel<__nv_bfloat16><<<grid_for(n, 256), 256, 0, st>>>(dQacc, (__nv_bfloat16 *)dQ, n, acc);
    }
    return launch_status();
}

}  // namespace

extern "C" {

size_t ssa_workspace_size(const ssa_dims_t *dims, int op) {
    Shape S;
    const bool need_k = op == SSA_OP_SPARSE_FWD || op == SSA_OP_SPARSE_BWD;
    if (check_dims(dims, S, need_k) != SSA_OK) return 0;
    return ws_bytes_for(S, op);
}

ssa_status_t ssa_block_pool(const ssa_dims_t *dims, const void *K, float *Kbar, ssa_stream_t stream) {
    Shape S;
    ssa_status_t e = check_dims(dims, S, false);
    if (e != SSA_OK) return e;
    if (!K || !Kbar) return SSA_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const size_t units = S.BHk * S.nb;  // one warp per (key/value head, block)
    const unsigned g = static_cast<unsigned>((units + kPoolWarps - 1) / kPoolWarps);
    const int blk = kPoolWarps * 32;
    if (S.dtype == SSA_DT_BF16) {
        if (S.d == 128)
            pool_kernel<__nv_bfloat16, 128><<<g, blk, 0, st>>>((const __nv_bfloat16 *)K, Kbar, S.T, S.s, S.nb, units);
        else
            pool_kernel<__nv_bfloat16, 64><<<g, blk, 0, st>>>((const __nv_bfloat16 *)K, Kbar, S.T, S.s, S.nb, units);
    } else {
        if (S.d == 128)
            pool_kernel<float, 128><<<g, blk, 0, st>>>((const float *)K, Kbar, S.T, S.s, S.nb, units);
        else
            pool_kernel<float, 64><<<g, blk, 0, st>>>((const float *)K, Kbar, S.T, S.s, S.nb, units);
    }
    return launch_status();
}

ssa_status_t ssa_block_select(const ssa_dims_t *dims, const void *Q, const float *Kbar, int32_t *idx,
                              unsigned flags, ssa_stream_t stream) {
    Shape S;
    ssa_status_t e = check_dims(dims, S, true);
    if (e != SSA_OK) return e;
    if (!Q || !Kbar || !idx) return SSA_ERR_INVALID_ARG;
    if (!(flags & SSA_SEL_FORCE_CURRENT) || (flags & ~static_cast<unsigned>(SSA_SEL_FORCE_CURRENT)))
        return SSA_ERR_UNSUPPORTED;
    const size_t sm = select_smem_bytes(S.d, S.nb);
    if (S.nb > 1024 || sm > 227 * 1024) return SSA_ERR_UNSUPPORTED;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (S.tc && S.nb <= kSelTcMaxBlocks) {
        // scores on the tensor cores
        const size_t smt = SelTcSmem::kTotal + 1024;
        if (!set_smem(select_tc_kernel, smt)) return SSA_ERR_CUDA;
        select_tc_kernel<<<dim3((S.T + kSelTcRows - 1) / kSelTcRows, S.BHk), kSelTcThreads, smt, st>>>(
            (const __nv_bfloat16 *)Q, Kbar, idx, S.T, S.s, S.k, S.nb, S.G);
        return launch_status();
    }
    if (S.dtype == SSA_DT_BF16) {
        if (S.nb <= 256)
            e = launch_select<__nv_bfloat16, 8>(S, Q, Kbar, idx, sm, st);
        else if (S.nb <= 512)
            e = launch_select<__nv_bfloat16, 16>(S, Q, Kbar, idx, sm, st);
        else
            e = launch_select<__nv_bfloat16, 32>(S, Q, Kbar, idx, sm, st);
    } else {
        if (S.nb <= 256)
            e = launch_select<float, 8>(S, Q, Kbar, idx, sm, st);
        else if (S.nb <= 512)
            e = launch_select<float, 16>(S, Q, Kbar, idx, sm, st);
        else
            e = launch_select<float, 32>(S, Q, Kbar, idx, sm, st);
    }
    if (e != SSA_OK) return e;
    return launch_status();
}

ssa_status_t ssa_sparse_index(const ssa_dims_t *dims, const int32_t *idx, void *index, size_t index_bytes_,
                              ssa_stream_t stream) {
    Shape S;
    ssa_status_t e = check_dims(dims, S, true);
    if (e != SSA_OK) return e;
    if (!idx) return SSA_ERR_INVALID_ARG;
    if (!S.tc) return SSA_OK;  // the CUDA-core kernels read idx directly
    if ((e = check_ws(S, SSA_OP_SPARSE_INDEX, index, index_bytes_)) != SSA_OK) return e;
    return build_index(S, idx, carve_index(S, index), reinterpret_cast<cudaStream_t>(stream));
}

ssa_status_t ssa_sparse_attn_fwd(const ssa_dims_t *dims, const void *Q, const void *K, const void *V,
                                 const int32_t *idx, const void *index, void *O, void *O_lo, float *lse, void *ws,
                                 size_t ws_bytes, ssa_stream_t stream) {
    Shape S;
    ssa_status_t e = check_dims(dims, S, true);
    if (e != SSA_OK) return e;
    if (!Q || !K || !V || !idx || !O || !lse) return SSA_ERR_INVALID_ARG;
    if ((e = check_ws(S, SSA_OP_SPARSE_FWD, ws, ws_bytes)) != SSA_OK) return e;
    if (index && (reinterpret_cast<uintptr_t>(index) & 15u)) return SSA_ERR_WORKSPACE;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (!S.tc) {
        if (S.dtype == SSA_DT_BF16)
            launch_simt_fwd<__nv_bfloat16>(S, Q, K, V, idx, O, O_lo, lse, st);
        else
            launch_simt_fwd<float>(S, Q, K, V, idx, O, O_lo, lse, st);
        return launch_status();
    }
    uint8_t *p = static_cast<uint8_t *>(ws);
    const IndexWs W = carve_index(S, index ? index : p);
    p += index_bytes(S);
    if (!index && (e = build_index(S, idx, W, st)) != SSA_OK) return e;
    const size_t nprow = S.BHk * list_stride(S.T, S.k, S.nb) * S.G;  // partial rows: G per list position
    __half *Opart = reinterpret_cast<__half *>(p);
    float *lsepart = reinterpret_cast<float *>(p + nprow * 128 * 2);
    p += align_up(nprow * (128 * 2 + 4));
    int32_t *bexp = reinterpret_cast<int32_t *>(p);  // [BHk * nb] exponents, then the "any set" flag
    if (cudaMemsetAsync(bexp + S.BHk * S.nb, 0, 4, st) != cudaSuccess) return SSA_ERR_CUDA;
    CUtensorMap tmK, tmV, tmO;
    // the fp16 partials are stored through a 16-bit tensor map (no conversion happens in a store)
    if (!make_tmap(&tmK, K, S.krows, S.s) || !make_tmap(&tmV, V, S.krows, S.s) ||
        !make_tmap(&tmO, Opart, nprow, 32))
        return SSA_ERR_CUDA;
    const unsigned units = static_cast<unsigned>(S.BHk * S.nb);
    const float sl2 = S.scale * kLog2e;
    auto run = [&](auto kernel, size_t sm) {
        if (!set_smem(kernel, sm)) return false;
        kernel<<<units, kSparseFwdThreads, sm, st>>>(tmK, tmV, tmO, (const __nv_bfloat16 *)Q, W.entries, W.lstart,
                                                     W.llen, W.order, lsepart, bexp, static_cast<int>(S.BHk), S.T, S.k, S.nb,
                                                     S.G, sl2);
        return true;
    };
    const bool gq = S.G > 1;
    const size_t sm128 = SparseFwdSmem<128>::kTotal + 1024, sm64 = SparseFwdSmem<64>::kTotal + 1024;
    const bool launched = S.s == 128 ? (gq ? run(sparse_fwd_kernel<128, true>, sm128) : run(sparse_fwd_kernel<128, false>, sm128))
                                     : (gq ? run(sparse_fwd_kernel<64, true>, sm64) : run(sparse_fwd_kernel<64, false>, sm64));
    if (!launched) return SSA_ERR_CUDA;
    const unsigned mg = static_cast<unsigned>((S.rows + 7) / 8);
    auto merge = [&](auto kernel) {
        kernel<<<mg, 256, 0, st>>>(W.pos, idx, bexp, Opart, lsepart, (__nv_bfloat16 *)O, (__nv_bfloat16 *)O_lo, lse,
                                   S.rows, S.T, S.k, S.nb, S.G);
    };
    if (S.k <= 8)
        merge(sparse_merge_kernel<1>);
    else if (S.k <= 16)
        merge(sparse_merge_kernel<2>);
    else if (S.k <= 32)
        merge(sparse_merge_kernel<4>);
    else
        merge(sparse_merge_kernel<0>);
    return launch_status();
}

ssa_status_t ssa_sparse_attn_bwd(const ssa_dims_t *dims, const void *Q, const void *K, const void *V,
                                 const void *O, const void *O_lo, const float *lse, const void *dO,
                                 const int32_t *idx, const void *index, void *dQ, void *dK, void *dV, int accumulate,
                                 void *ws, size_t ws_bytes, ssa_stream_t stream) {
    Shape S;
    ssa_status_t e = check_dims(dims, S, true);
    if (e != SSA_OK) return e;
    if (!Q || !K || !V || !O || !lse || !dO || !idx || !dQ || !dK || !dV) return SSA_ERR_INVALID_ARG;
    if ((e = check_grads(accumulate, dQ, dK, dV)) != SSA_OK) return e;
    if ((e = check_ws(S, SSA_OP_SPARSE_BWD, ws, ws_bytes)) != SSA_OK) return e;
    if (index && (reinterpret_cast<uintptr_t>(index) & 15u)) return SSA_ERR_WORKSPACE;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (S.tc) return tc_bwd(S, Q, K, V, O, O_lo, lse, dO, idx, index, dQ, dK, dV, accumulate, ws, st);
    if (S.dtype == SSA_DT_BF16)
        return simt_bwd<__nv_bfloat16>(S, Q, K, V, O, O_lo, lse, dO, idx, dQ, dK, dV, accumulate, ws, st);
    return simt_bwd<float>(S, Q, K, V, O, O_lo, lse, dO, idx, dQ, dK, dV, accumulate, ws, st);
}

ssa_status_t ssa_full_attn_fwd(const ssa_dims_t *dims, const void *Q, const void *K, const void *V, void *O,
                               void *O_lo, float *lse, void *ws, size_t ws_bytes, ssa_stream_t stream) {
    Shape S;
    ssa_status_t e = check_dims(dims, S, false);
    if (e != SSA_OK) return e;
    if (!Q || !K || !V || !O || !lse) return SSA_ERR_INVALID_ARG;
    (void)ws;
    (void)ws_bytes;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (!S.tc) {
        if (S.dtype == SSA_DT_BF16)
            launch_simt_fwd<__nv_bfloat16>(S, Q, K, V, nullptr, O, O_lo, lse, st);
        else
            launch_simt_fwd<float>(S, Q, K, V, nullptr, O, O_lo, lse, st);
        return launch_status();
    }
    CUtensorMap tmQ, tmK, tmV;
    if (!make_tmap(&tmQ, Q, S.rows, 128) || !make_tmap(&tmK, K, S.krows, 128) || !make_tmap(&tmV, V, S.krows, 128))
        return SSA_ERR_CUDA;
    const size_t sm = FullFwdSmem::kTotal + 1024;
    if (!set_smem(full_fwd_kernel, sm)) return SSA_ERR_CUDA;
    const unsigned grid = static_cast<unsigned>(S.BH * ((S.T + 255) / 256));
    full_fwd_kernel<<<grid, kFullFwdThreads, sm, st>>>(tmQ, tmK, tmV, (__nv_bfloat16 *)O, (__nv_bfloat16 *)O_lo, lse,
                                                      static_cast<int>(S.BH), S.T, S.G, S.scale * kLog2e);
    return launch_status();
}

ssa_status_t ssa_full_attn_bwd(const ssa_dims_t *dims, const void *Q, const void *K, const void *V,
                               const void *O, const void *O_lo, const float *lse, const void *dO, void *dQ, void *dK,
                               void *dV, int accumulate, void *ws, size_t ws_bytes, ssa_stream_t stream) {
    Shape S;
    ssa_status_t e = check_dims(dims, S, false);
    if (e != SSA_OK) return e;
    if (!Q || !K || !V || !O || !lse || !dO || !dQ || !dK || !dV) return SSA_ERR_INVALID_ARG;
    if ((e = check_grads(accumulate, dQ, dK, dV)) != SSA_OK) return e;
    if ((e = check_ws(S, SSA_OP_FULL_BWD, ws, ws_bytes)) != SSA_OK) return e;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (S.tc) return tc_bwd(S, Q, K, V, O, O_lo, lse, dO, nullptr, nullptr, dQ, dK, dV, accumulate, ws, st);
    if (S.dtype == SSA_DT_BF16)
        return simt_bwd<__nv_bfloat16>(S, Q, K, V, O, O_lo, lse, dO, nullptr, dQ, dK, dV, accumulate, ws, st);
    return simt_bwd<float>(S, Q, K, V, O, O_lo, lse, dO, nullptr, dQ, dK, dV, accumulate, ws, st);
}

ssa_status_t ssa_align_loss_fwd(const ssa_dims_t *dims, const void *Of, const void *Os, int kind, float beta,
                                float w_sparsity, float w_commit, float *loss_dev, void *ws, size_t ws_bytes,
                                ssa_stream_t stream) {
    Shape S;
    ssa_status_t e = check_dims(dims, S, false);
    if (e != SSA_OK) return e;
    if (!Of || !Os || !loss_dev) return SSA_ERR_INVALID_ARG;
    if (kind != SSA_ALIGN_SMOOTH_L1 && kind != SSA_ALIGN_L2) return SSA_ERR_INVALID_ARG;
    if (!(beta > 0.f) || !std::isfinite(beta) || !std::isfinite(w_sparsity) || !std::isfinite(w_commit))
        return SSA_ERR_INVALID_ARG;
    if ((e = check_ws(S, SSA_OP_ALIGN_FWD, ws, ws_bytes)) != SSA_OK) return e;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    float *partial = static_cast<float *>(ws);
    const size_t n = S.rows * S.d;
    if (S.dtype == SSA_DT_BF16)
        align_fwd_partial_kernel<__nv_bfloat16><<<kAlignBlocks, 256, 0, st>>>(
            (const __nv_bfloat16 *)Of, (const __nv_bfloat16 *)Os, partial, n, kind, beta);
    else
        align_fwd_partial_kernel<float><<<kAlignBlocks, 256, 0, st>>>((const float *)Of, (const float *)Os, partial,
                                                                      n, kind, beta);
    align_fwd_final_kernel<<<1, 32, 0, st>>>(partial, kAlignBlocks, loss_dev,
                                             (static_cast<double>(w_sparsity) + w_commit) / static_cast<double>(n));
    return launch_status();
}

ssa_status_t ssa_align_loss_bwd(const ssa_dims_t *dims, const void *Of, const void *Os, int kind, float beta,
                                float w_sparsity, float w_commit, const float *dloss_dev, void *dOf, void *dOs,
                                int accumulate, ssa_stream_t stream) {
    Shape S;
    ssa_status_t e = check_dims(dims, S, false);
    if (e != SSA_OK) return e;
    if (!Of || !Os || !dloss_dev || !dOf || !dOs) return SSA_ERR_INVALID_ARG;
    if (kind != SSA_ALIGN_SMOOTH_L1 && kind != SSA_ALIGN_L2) return SSA_ERR_INVALID_ARG;
    if (!(beta > 0.f) || !std::isfinite(beta) || !std::isfinite(w_sparsity) || !std::isfinite(w_commit))
        return SSA_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const size_t n = S.rows * S.d;
    if (S.dtype == SSA_DT_BF16)
        align_bwd_kernel<__nv_bfloat16><<<grid_for(n, 256), 256, 0, st>>>(
            (const __nv_bfloat16 *)Of, (const __nv_bfloat16 *)Os, dloss_dev, (__nv_bfloat16 *)dOf,
            (__nv_bfloat16 *)dOs, n, kind, beta, w_sparsity, w_commit, accumulate);
    else
        align_bwd_kernel<float><<<grid_for(n, 256), 256, 0, st>>>((const float *)Of, (const float *)Os, dloss_dev,
                                                                  (float *)dOf, (float *)dOs, n, kind, beta,
                                                                  w_sparsity, w_commit, accumulate);
    return launch_status();
}

ssa_status_t ssa_dropped_mass(const ssa_dims_t *dims, const float *lse_sparse, const float *lse_full, float *delta,
                              ssa_stream_t stream) {
    Shape S;
    ssa_status_t e = check_dims(dims, S, false);
    if (e != SSA_OK) return e;
    if (!lse_sparse || !lse_full || !delta) return SSA_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    dropped_mass_kernel<<<grid_for(S.rows, 256), 256, 0, st>>>(lse_sparse, lse_full, delta, S.rows);
    return launch_status();
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free full attention backward: scratch in a static device array.
// In host code the array's name is only a stand-in; its device address comes
// from cudaGetSymbolAddress, looked up with the caller's device current.
// ---------------------------------------------------------------------------
static __device__ __align__(256) unsigned char g_noalloc_scratch[SSA_NOALLOC_SCRATCH_BYTES];

namespace {
// Device address of the scratch array in the current device's context.  Looked up on
// every call (the lookup allocates nothing): an address cached across calls would be
// stale after the context is torn down and the module loaded again.
ssa_status_t noalloc_scratch(void **out) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return SSA_ERR_CUDA;
    *out = p;
    return SSA_OK;
}

// One slot's block of the decode against the G query heads, for G padded to GP.
template <int GP>
bool launch_decode_attend(const Shape &S, cudaStream_t st, const int32_t *cache_len, const void *q, const void *Kc,
                          const void *Vc, const int32_t *idx, float *opart, float *lsepart) {
    const size_t sm = dec_attend_smem(S.s, GP);
    if (!set_smem(decode_attend_kernel<GP>, sm)) return false;
    decode_attend_kernel<GP><<<dim3(static_cast<unsigned>(S.BHk), S.k), kDecThreads, sm, st>>>(
        cache_len, (const __nv_bfloat16 *)q, (const __nv_bfloat16 *)Kc, (const __nv_bfloat16 *)Vc, idx, opart, lsepart,
        S.Hk, S.G, S.T, S.s, S.k, S.scale);
    return true;
}
}  // namespace

extern "C" {

ssa_status_t ssa_full_attn_bwd_noalloc(const ssa_dims_t *dims, const void *Q, const void *K, const void *V,
                                       const void *O, const void *O_lo, const float *lse, const void *dO, void *dQ,
                                       void *dK, void *dV, int accumulate, ssa_stream_t stream) {
    Shape S;
    ssa_status_t e = check_dims(dims, S, false);
    if (e != SSA_OK) return e;
    if (!Q || !K || !V || !O || !lse || !dO || !dQ || !dK || !dV) return SSA_ERR_INVALID_ARG;
    const size_t need = ws_bytes_for(S, SSA_OP_FULL_BWD);
    if (need > SSA_NOALLOC_SCRATCH_BYTES) return SSA_ERR_WORKSPACE;
    void *ws = nullptr;
    if ((e = noalloc_scratch(&ws)) != SSA_OK) return e;
    return ssa_full_attn_bwd(dims, Q, K, V, O, O_lo, lse, dO, dQ, dK, dV, accumulate, ws, SSA_NOALLOC_SCRATCH_BYTES,
                             stream);
}

ssa_status_t ssa_sparse_decode(const ssa_dims_t *dims, const int32_t *cache_len, const void *q, const void *Kcache,
                               const void *Vcache, float *Kbar_cache, int32_t *idx, void *o, float *lse, void *ws,
                               size_t ws_bytes, ssa_stream_t stream) {
    Shape S;
    ssa_status_t e = check_dims(dims, S, true);
    if (e != SSA_OK) return e;
    if (!cache_len || !q || !Kcache || !Vcache || !Kbar_cache || !idx || !o || !lse) return SSA_ERR_INVALID_ARG;
    if (S.dtype != SSA_DT_BF16 || S.d != 128 || S.nb > kDecMaxBlocks || S.G > kDecMaxGroup) return SSA_ERR_UNSUPPORTED;
    // the selected blocks are bulk-copied and the query rows read in 16-byte units: 16-byte aligned bases
    if ((reinterpret_cast<uintptr_t>(Kcache) | reinterpret_cast<uintptr_t>(Vcache) | reinterpret_cast<uintptr_t>(q)) &
        15u)
        return SSA_ERR_INVALID_ARG;
    if ((e = check_ws(S, SSA_OP_DECODE, ws, ws_bytes)) != SSA_OK) return e;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    float *opart = static_cast<float *>(ws);
    float *lsepart = reinterpret_cast<float *>(static_cast<uint8_t *>(ws) + align_up(S.BH * S.k * S.d * 4));
    const unsigned bhk = static_cast<unsigned>(S.BHk);
    const size_t sm = (128 + (S.nb > 256 ? S.nb : 256)) * sizeof(float);
    // the warp search holds ceil(nb / 32) scores per lane (8, 16 or 32)
    auto sel = S.nb <= 256 ? decode_select_kernel<8> : S.nb <= 512 ? decode_select_kernel<16> : decode_select_kernel<32>;
    sel<<<bhk, kDecThreads, sm, st>>>(cache_len, (const __nv_bfloat16 *)q, (const __nv_bfloat16 *)Kcache, Kbar_cache,
                                      idx, S.Hk, S.G, S.T, S.s, S.k, S.nb);
    if (S.s == 128) {  // tensor-core attend: blocks brought in by TMA, both products on tcgen05
        CUtensorMap tmK, tmV;
        if (!make_tmap(&tmK, Kcache, S.krows, 128) || !make_tmap(&tmV, Vcache, S.krows, 128)) return SSA_ERR_CUDA;
        if (!set_smem(decode_attend_tc_kernel, DecTcSmem::kTotal)) return SSA_ERR_CUDA;
        decode_attend_tc_kernel<<<dim3(bhk, S.k), 128, DecTcSmem::kTotal, st>>>(
            tmK, tmV, cache_len, (const __nv_bfloat16 *)q, idx, opart, lsepart, S.Hk, S.G, S.T, S.k,
            S.scale * 1.4426950408889634f);
    } else {  // blocks of 64 keys: CUDA-core attend, the group padded to a power of two
        auto launch = S.G <= 1   ? launch_decode_attend<1>
                      : S.G <= 2 ? launch_decode_attend<2>
                      : S.G <= 4 ? launch_decode_attend<4>
                      : S.G <= 8 ? launch_decode_attend<8>
                                 : launch_decode_attend<16>;
        if (!launch(S, st, cache_len, q, Kcache, Vcache, idx, opart, lsepart)) return SSA_ERR_CUDA;
    }
    const unsigned rows = static_cast<unsigned>(S.BH);
    decode_combine_kernel<<<(rows + kDecThreads / 32 - 1) / (kDecThreads / 32), kDecThreads, 0, st>>>(
        opart, lsepart, (__nv_bfloat16 *)o, lse, static_cast<int>(rows), S.k);
    return launch_status();
}

ssa_status_t ssa_rope(const ssa_dims_t *dims, void *X, int heads, int pos0, float base, float factor, int transpose,
                      ssa_stream_t stream) {
    Shape S;
    ssa_status_t e = check_dims(dims, S, false);
    if (e != SSA_OK) return e;
    if (!X || heads < 1 || pos0 < 0 || !(base > 1.f) || !std::isfinite(base) || !(factor > 0.f) ||
        !std::isfinite(factor))
        return SSA_ERR_INVALID_ARG;
    if (static_cast<size_t>(S.B) * heads * S.T > 0x7FFFFFFFull) return SSA_ERR_UNSUPPORTED;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const dim3 grid((S.T + kRopeRows - 1) / kRopeRows, S.B);
    const double l2b = std::log2(static_cast<double>(base)), inv = 1.0 / static_cast<double>(factor);
    if (S.dtype == SSA_DT_BF16)
        rope_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>((__nv_bfloat16 *)X, heads, S.T, S.d, pos0, l2b, inv,
                                                         transpose ? 1 : 0);
    else
        rope_kernel<float><<<grid, 256, 0, st>>>((float *)X, heads, S.T, S.d, pos0, l2b, inv, transpose ? 1 : 0);
    return launch_status();
}

ssa_status_t ssa_wait_probe(uint64_t limit_ns, ssa_stream_t stream) {
    if (limit_ns < 1000u || limit_ns > 1000000000u) return SSA_ERR_INVALID_ARG;
    wait_probe_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(limit_ns);
    return launch_status();
}

ssa_status_t ssa_get_device_error(ssa_stream_t stream) {
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(st) != cudaSuccess) return SSA_ERR_CUDA;
    unsigned int w = 0;
    if (cudaMemcpyFromSymbol(&w, g_error_word, sizeof(w)) != cudaSuccess) return SSA_ERR_CUDA;
    if (w == 0) return SSA_OK;
    const unsigned int zero = 0;
    if (cudaMemcpyToSymbol(g_error_word, &zero, sizeof(zero)) != cudaSuccess) return SSA_ERR_CUDA;
    return (w >> 24) == ERR_BAD_INPUT ? SSA_ERR_BAD_INPUT : SSA_ERR_TIMEOUT;
}

const char *ssa_status_string(ssa_status_t s) {
    switch (s) {
        case SSA_OK: return "SSA_OK";
        case SSA_ERR_INVALID_ARG: return "SSA_ERR_INVALID_ARG";
        case SSA_ERR_UNSUPPORTED: return "SSA_ERR_UNSUPPORTED";
        case SSA_ERR_WORKSPACE: return "SSA_ERR_WORKSPACE";
        case SSA_ERR_CUDA: return "SSA_ERR_CUDA";
        case SSA_ERR_TIMEOUT: return "SSA_ERR_TIMEOUT";
        case SSA_ERR_BAD_INPUT: return "SSA_ERR_BAD_INPUT";
    }
    return "SSA_ERR_UNKNOWN";
}

}  // extern "C"
