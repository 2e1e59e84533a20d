// attn_bwd.cuh -- tcgen05 attention backward shared by the full and the sparse
// stream (head dimension 128, bf16 inputs, fp32 accumulation).
//
// Key-block-outer: one CTA per key tile (full: 128 keys; the query tiles from
// the diagonal on) or per key block j (sparse: s keys; the 128-row tiles of the
// queries whose selection holds j, gathered by row).  K_j, V_j stay in shared
// memory and the transposed accumulators dV_j^T, dK_j^T stay in tensor memory
// for the whole unit.  Per query tile:
//   S = Q K^T, dP = dO V^T                      (M = 128 query rows)
//   P = exp(scale S - lse), dS = P o (dP - D)   -> shared memory, bf16
//   dV^T += dO^T P, dK^T += Q^T dS              (M = head dim 128)
//   dQ = dS K                                    -> fp32 vector atomics, * scale
// Paper: section 4.2 (keys outside S(t) get no gradient; the selection is a
// constant), FlashAttention-2 style recomputation of P from the saved lse.
//
// Warp roles (320 threads):
//   warps 0-7  two warpgroups; warp w owns query row (w & 3)*32 + lane and
//              column half (w >> 2) of every row-wise phase;
//   warp 8     MMA issuer (one thread);
//   warp 9     TMA producer (K_j, V_j; contiguous Q / dO tiles of the full stream).
// Overlap: Q/dO of the next tile are loaded as soon as the dV/dK MMAs of the
// current tile have consumed them; dQ leaves tensor memory before its atomics,
// so the next tile's S/dP MMAs run while the atomics drain.
//
// Shared memory: Q 32 KB | dO 32 KB | K, V NKV*256 B each | P, dS (NKV/64)*16 KB each
// Tensor memory: S / dQ at column 0, dP at 128, dV^T at 256, dK^T at 384 (512).
#pragma once

#include "attn_tc.cuh"

namespace ssa {

template <int NKV>
struct BwdSmem {
    static constexpr int kQ = 0;
    static constexpr int kdO = kQ + 2 * kChunkBytes;
    static constexpr int kK = kdO + 2 * kChunkBytes;
    static constexpr int kV = kK + 2 * NKV * 128;
    static constexpr int kP = kV + 2 * NKV * 128;
    static constexpr int kdS = kP + (NKV / 64) * kChunkBytes;
    static constexpr int kBar = kdS + (NKV / 64) * kChunkBytes;
    static constexpr int kTotal = kBar + 256;
};

struct BwdArgs {
    const __nv_bfloat16 *Q, *dO;
    const float *lse, *Dvec;
    float *dQacc;
    __nv_bfloat16 *dK, *dV;
    const int32_t *entries, *lstart, *llen;  // sparse only
    int BH, T, k, nb, sparse, accumulate;
    float scale, scale_log2;
};

constexpr int kBwdThreads = 320;

template <int NKV>
__global__ void __launch_bounds__(kBwdThreads, 1)
    attn_bwd_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                    const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmdO,
                    const BwdArgs a) {
    using L = BwdSmem<NKV>;
    constexpr int HALF = NKV / 2;  // S / dP columns per warpgroup
    // 128-key units stage the dQ tile (64 KB) through the P / dS buffers and add it
    // with coalesced row reductions; 64-key units (buffers of 32 KB) add per row.
    constexpr bool kCoalescedFlush = NKV == 128;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::kBar);
    uint64_t *bar_kv = bars + 0, *bar_qdo_full = bars + 1, *bar_sdp_full = bars + 2, *bar_pds_full = bars + 3;
    uint64_t *bar_qdo_free = bars + 4, *bar_dq_full = bars + 5, *bar_dq_empty = bars + 6, *bar_final = bars + 7;
    uint64_t *bar_staged = bars + 8, *bar_flushed = bars + 9;  // dQ staging in the P / dS buffers
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 10);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(bars + 11);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int T = a.T;
    // Head-major unit order, heaviest key block of each head first: the query
    // rows and the dQ accumulator of the head being worked on stay in L2.
    const int units_per_head = a.sparse ? a.nb : (a.T + NKV - 1) / NKV;
    const int bh = blockIdx.x / units_per_head, kb = blockIdx.x % units_per_head;
    const int kv0 = kb * NKV;
    const size_t head_rows = static_cast<size_t>(bh) * T;
    const bool sparse = a.sparse != 0;
    Rows R;
    if (sparse) {
        R.list = a.entries + static_cast<size_t>(bh) * list_stride(T, a.k, a.nb) + a.lstart[bh * a.nb + kb];
        R.len = a.llen[bh * a.nb + kb];
        R.first = 0;
    } else {
        R.list = nullptr;
        R.first = kv0;  // causal: query tiles from the key tile onward
        R.len = T - kv0;
    }
    R.k = a.k;
    const int ntiles = (R.len + kTileQ - 1) / kTileQ;

    const uint32_t sQ = smem_u32(smem + L::kQ), sdO = smem_u32(smem + L::kdO), sK = smem_u32(smem + L::kK),
                   sV = smem_u32(smem + L::kV), sP = smem_u32(smem + L::kP), sdS = smem_u32(smem + L::kdS);

    if (threadIdx.x == 0) {
        mbar_init(bar_kv, 1);
        mbar_init(bar_qdo_full, sparse ? 256 : 1);
        mbar_init(bar_sdp_full, 1);
        mbar_init(bar_pds_full, 256);
        mbar_init(bar_qdo_free, 1);
        mbar_init(bar_dq_full, 1);
        mbar_init(bar_dq_empty, 256);
        mbar_init(bar_final, 1);
        mbar_init(bar_staged, 256);
        mbar_init(bar_flushed, 256);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tS = tmem, tdP = tmem + 128, tdV = tmem + 256, tdK = tmem + 384, tdQ = tmem;

    if (warp == 9) {
        // ---------------- TMA producer ----------------
        if (lane == 0) {
            const int krow = static_cast<int>(head_rows) + kv0;
            mbar_arrive_expect_tx(bar_kv, 4 * NKV * 128);
            tma_load_2d(&tmK, bar_kv, smem + L::kK, 0, krow);
            tma_load_2d(&tmK, bar_kv, smem + L::kK + NKV * 128, 64, krow);
            tma_load_2d(&tmV, bar_kv, smem + L::kV, 0, krow);
            tma_load_2d(&tmV, bar_kv, smem + L::kV + NKV * 128, 64, krow);
            if (!sparse) {
                for (int it = 0; it < ntiles; ++it) {
                    if (it > 0 && !mbar_wait(bar_qdo_free, (it - 1) & 1, abort_flag, 0x311)) break;
                    const int qrow = static_cast<int>(head_rows) + kv0 + it * kTileQ;
                    mbar_arrive_expect_tx(bar_qdo_full, 4 * kChunkBytes);
                    tma_load_2d(&tmQ, bar_qdo_full, smem + L::kQ, 0, qrow);
                    tma_load_2d(&tmQ, bar_qdo_full, smem + L::kQ + kChunkBytes, 64, qrow);
                    tma_load_2d(&tmdO, bar_qdo_full, smem + L::kdO, 0, qrow);
                    tma_load_2d(&tmdO, bar_qdo_full, smem + L::kdO + kChunkBytes, 64, qrow);
                }
            }
        }
    } else if (warp == 8) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            const uint32_t idS = idesc_bf16(128, NKV, false, false);  // S, dP
            const uint32_t idT = idesc_bf16(128, NKV, true, true);    // dV^T, dK^T
            const uint32_t idQ = idesc_bf16(128, 128, false, true);   // dQ
            bool ok = mbar_wait(bar_kv, 0, abort_flag, 0x301);
            for (int it = 0; ok && it < ntiles; ++it) {
                if (!mbar_wait(bar_qdo_full, it & 1, abort_flag, 0x302)) break;
                if (it > 0 && !mbar_wait(bar_dq_empty, (it - 1) & 1, abort_flag, 0x303)) break;
                tc_fence_after();
                mma_k128_kmajor(tS, sQ, sK, NKV * 128, idS);
                mma_k128_kmajor(tdP, sdO, sV, NKV * 128, idS);
                mma_commit(bar_sdp_full);
                if (!mbar_wait(bar_pds_full, it & 1, abort_flag, 0x304)) break;
                tc_fence_after();
                // dV^T[d x kv] += dO^T P ; dK^T[d x kv] += Q^T dS   (K = 128 query rows)
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    mma_bf16_ss(tdV, smem_desc_sw128(sdO + kk * 2048, kChunkBytes),
                                smem_desc_sw128(sP + kk * 2048, kChunkBytes), idT, (it > 0 || kk > 0) ? 1u : 0u);
                }
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    mma_bf16_ss(tdK, smem_desc_sw128(sQ + kk * 2048, kChunkBytes),
                                smem_desc_sw128(sdS + kk * 2048, kChunkBytes), idT, (it > 0 || kk > 0) ? 1u : 0u);
                }
                mma_commit(bar_qdo_free);
                // dQ[q x d] = dS K   (K = NKV keys)
#pragma unroll
                for (int kk = 0; kk < NKV / 16; ++kk) {
                    mma_bf16_ss(tdQ, smem_desc_sw128(sdS + (kk >> 2) * kChunkBytes + (kk & 3) * 32, 16),
                                smem_desc_sw128(sK + kk * 2048, NKV * 128), idQ, kk > 0 ? 1u : 0u);
                }
                mma_commit(bar_dq_full);
            }
            mma_commit(bar_final);
            mbar_wait(bar_final, 0, abort_flag, 0x305);
        }
    } else {
        // ---------------- compute warps ----------------
        const int r = ((warp & 3) << 5) | lane;  // tile row
        const int h = warp >> 2;                 // column half
        const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
        int t = 0, e = 0;
        bool valid = ntiles > 0 && tile_row(R, T, 0, r, t, e);
        if (sparse) {
            // warpgroup 0 gathers Q rows, warpgroup 1 dO rows
            const __nv_bfloat16 *src = (h == 0 ? a.Q : a.dO) + (head_rows + (valid ? t : 0)) * kD;
            gather_row(h == 0 ? sQ : sdO, src, valid, r);
            cp_async_commit();
            cp_async_wait_all();
            fence_proxy_async_smem();
            mbar_arrive(bar_qdo_full);
        }
        bool ok = true;
        for (int it = 0; it < ntiles; ++it) {
            const float lse2 = valid ? __ldg(a.lse + head_rows + t) * kLog2e : 0.f;
            const float Dt = valid ? __ldg(a.Dvec + head_rows + t) : 0.f;
            if (!mbar_wait(bar_sdp_full, it & 1, abort_flag, 0x306)) {
                ok = false;
                break;
            }
            tc_fence_after();
            // the previous tile's dQ flush staged through P / dS: wait until it has read them
            if (kCoalescedFlush && it > 0 && !mbar_wait(bar_flushed, (it - 1) & 1, abort_flag, 0x309)) {
                ok = false;
                break;
            }
            // all tensor-memory loads of this row half in flight at once, one wait
            uint32_t sraw[HALF / 32][32], draw[HALF / 32][32];
#pragma unroll
            for (int c = 0; c < HALF / 32; ++c) {
                tmem_ld32_async(tS + lane_off + h * HALF + 32 * c, sraw[c]);
                tmem_ld32_async(tdP + lane_off + h * HALF + 32 * c, draw[c]);
            }
            tmem_ld_wait();
            // key kv0 + col is attended when col <= lim (causal inside the diagonal block)
            const int lim = valid ? t - kv0 - h * HALF : -1;
#pragma unroll
            for (int c = 0; c < HALF / 32; ++c) {
                float sv[32], dp[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const float p = (32 * c + i <= lim)
                                        ? fast_exp2(fmaf(__uint_as_float(sraw[c][i]), a.scale_log2, -lse2))
                                        : 0.f;
                    sv[i] = p;
                    dp[i] = p * (__uint_as_float(draw[c][i]) - Dt);
                }
                store_row32_bf16(sP, kChunkBytes, r, h * HALF + 32 * c, sv);
                store_row32_bf16(sdS, kChunkBytes, r, h * HALF + 32 * c, dp);
            }
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(bar_pds_full);
            // next tile's rows (sparse: gathered by these threads once Q/dO are consumed)
            int t_next = 0, e_next = 0;
            bool valid_next = false;
            const bool more = it + 1 < ntiles;
            if (more) valid_next = tile_row(R, T, it + 1, r, t_next, e_next);
            if (sparse && more) {
                if (!mbar_wait(bar_qdo_free, it & 1, abort_flag, 0x308)) {
                    ok = false;
                    break;
                }
                const __nv_bfloat16 *src = (h == 0 ? a.Q : a.dO) + (head_rows + (valid_next ? t_next : 0)) * kD;
                gather_row(h == 0 ? sQ : sdO, src, valid_next, r);
                cp_async_commit();
            }
            if (!mbar_wait(bar_dq_full, it & 1, abort_flag, 0x307)) {
                ok = false;
                break;
            }
            tc_fence_after();
            uint32_t g[2][32];
            tmem_ld32_async(tdQ + lane_off + h * 64, g[0]);
            tmem_ld32_async(tdQ + lane_off + h * 64 + 32, g[1]);
            tmem_ld_wait();
            tc_fence_before();
            mbar_arrive(bar_dq_empty);
            if constexpr (kCoalescedFlush) {
                // Stage the tile's dQ rows (fp32, 512 B per row, 16-byte units XOR-swizzled by
                // row) in the P / dS buffers, free once every MMA of this tile has completed;
                // then each warp adds 16 whole rows with coalesced float4 reductions.
                auto stage_addr = [&](int row, int unit) -> uint32_t {
                    const uint32_t base = row < 64 ? sP + row * 512 : sdS + (row - 64) * 512;
                    return base + (((unit ^ row) & 31) << 4);
                };
#pragma unroll
                for (int q = 0; q < 16; ++q) {
                    const uint32_t *x = g[q >> 3] + 4 * (q & 7);
                    st_shared_v4(stage_addr(r, 16 * h + q), __float_as_uint(__uint_as_float(x[0]) * a.scale),
                                 __float_as_uint(__uint_as_float(x[1]) * a.scale),
                                 __float_as_uint(__uint_as_float(x[2]) * a.scale),
                                 __float_as_uint(__uint_as_float(x[3]) * a.scale));
                }
                mbar_arrive(bar_staged);
                if (!mbar_wait(bar_staged, it & 1, abort_flag, 0x30a)) {
                    ok = false;
                    break;
                }
                const int t_mine = valid ? t : -1;
#pragma unroll 4
                for (int i = 0; i < 16; ++i) {
                    const int row = 32 * (warp & 3) + 16 * h + i;
                    const int t_dst = __shfl_sync(0xffffffffu, t_mine, 16 * h + i);
                    if (t_dst >= 0) {
                        float4 v;
                        asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                                     : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                                     : "r"(stage_addr(row, lane)));
                        atomicAdd(reinterpret_cast<float4 *>(a.dQacc + (head_rows + t_dst) * kD) + lane, v);
                    }
                }
                mbar_arrive(bar_flushed);
            } else if (valid) {
                float4 *dq = reinterpret_cast<float4 *>(a.dQacc + (head_rows + t) * kD + h * 64);
#pragma unroll
                for (int q = 0; q < 16; ++q) {
                    const uint32_t *x = g[q >> 3] + 4 * (q & 7);
                    atomicAdd(dq + q, make_float4(__uint_as_float(x[0]) * a.scale, __uint_as_float(x[1]) * a.scale,
                                                  __uint_as_float(x[2]) * a.scale, __uint_as_float(x[3]) * a.scale));
                }
            }
            if (sparse && more) {
                cp_async_wait_all();
                fence_proxy_async_smem();
                mbar_arrive(bar_qdo_full);
            }
            t = t_next;
            e = e_next;
            valid = valid_next;
        }
        cp_async_wait_all();
        // Epilogue: thread <-> head-dim row r of dV^T / dK^T, key columns of its half.
        if (ok) {
#pragma unroll
            for (int c0 = h * HALF; c0 < (h + 1) * HALF; c0 += 32) {
                uint32_t rv[32], rk[32];
                tmem_ld32_async(tdV + lane_off + c0, rv);
                tmem_ld32_async(tdK + lane_off + c0, rk);
                tmem_ld_wait();
                float gv[32], gk[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    gv[i] = __uint_as_float(rv[i]);
                    gk[i] = __uint_as_float(rk[i]);
                }
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int kv = kv0 + c0 + i;
                    if (kv < T) {
                        const size_t off = (head_rows + kv) * kD + r;
                        float vv = ntiles > 0 ? gv[i] : 0.f, kk = ntiles > 0 ? gk[i] * a.scale : 0.f;
                        if (a.accumulate) {
                            vv += __bfloat162float(a.dV[off]);
                            kk += __bfloat162float(a.dK[off]);
                        }
                        a.dV[off] = __float2bfloat16_rn(vv);
                        a.dK[off] = __float2bfloat16_rn(kk);
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, 512);
}

}  // namespace ssa
