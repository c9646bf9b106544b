// Fused row-LSE + block-energy pass for sm_100a.
//
// Block energy: split the post-softmax attention matrix P into B x B blocks and sum each
// one (summaries of "Accelerating Text-to-Video Generation with Calibrated Sparse
// Attention": [zh] §2.2A, [de] §2A.1, [pt] §2A.2, [fr] §2.A and §2.B.1).  P is never
// stored:  E[h,i,j] = sum_{r in I_i} sum_{c in J_j} 2^(x_rc - lse2_r),  x = s * scale*log2(e),
// lse2 = LSE / ln 2.
//
// One CTA per (head h, query block i), 192 threads:
//   warp 0      TMA: Q tile (unless the rows are gathered), then K_j for every key block,
//               twice when the LSE is not supplied (pass 1 computes it, pass 2 sums).
//   warp 1      TMEM owner (256 columns: two S buffers) and MMA issuer, S = Q K_j^T.
//   warps 2..5  one row per thread: pass 1 keeps an exact running max / sum and ends with
//               the row's LSE in a register (the LSE is never written to memory, so no
//               scratch buffer is needed); pass 2 sums 2^(x - lse2) over the tile's valid
//               columns, reduces the 128 rows (warp shuffles, then 4 partials in fixed
//               order) and writes one energy per tile.
// [AdaSpa] §2 caches the LSE to reuse it in a later search; a supplied LSE skips pass 1.
#pragma once
#include <cuda_bf16.h>
#include "ptx.cuh"
#include "attn_fwd.cuh"

namespace calib {

constexpr uint32_t kEnergyTmemCols = 256;
constexpr int kEnergyThreads = 192;

struct EnergyParams {
    const __nv_bfloat16* q;   // [H, N, D] (read directly only for gathered rows)
    const int32_t* q_rows;    // [n_q] token indices or nullptr
    const float* lse_in;      // [H, Nq] natural-log LSE or nullptr
    float* energy;            // [H, nq, nk]
    int H, N, Nq, nq, nk;
    int accumulate;
    float scale_log2;
    uint64_t timeout_ns;
};

template <int D, int BLK, int KST>
struct EnergySmem {
    static constexpr int CH = D / 64;
    static constexpr uint32_t Q_BYTES = CH * kTileM * 128;
    static constexpr uint32_t K_BYTES = CH * BLK * 128;
    static constexpr uint32_t OFF_K = Q_BYTES;
    static constexpr uint32_t OFF_BAR = OFF_K + KST * K_BYTES;
    static constexpr int B_Q = 0, B_KF = 1, B_KE = B_KF + KST, B_SF = B_KE + KST, B_SE = B_SF + 2,
                         B_DRAIN = B_SE + 2, NBARS = B_DRAIN + 1;
    static constexpr uint32_t OFF_RED = OFF_BAR + NBARS * 8;      // float red[2][4]
    static constexpr uint32_t OFF_MISC = OFF_RED + 32;
    // at least 80 KB: two CTAs of 256 TMEM columns each per SM
    static constexpr uint32_t RAW = OFF_MISC + 16 + 1024;
    static constexpr uint32_t BYTES = RAW > 80u * 1024 ? RAW : 80u * 1024;
};

template <int D, int BLK, int KST>
__global__ void __launch_bounds__(kEnergyThreads, 1)
block_energy_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const EnergyParams p) {
    using L = EnergySmem<D, BLK, KST>;
    constexpr int CH = L::CH;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    uint8_t* sQ = smem;
    uint8_t* sK = smem + L::OFF_K;
    const uint32_t bar0 = smem_u32(smem + L::OFF_BAR);
    auto bar = [&](int idx) -> uint32_t { return bar0 + 8u * idx; };
    float* red = reinterpret_cast<float*>(smem + L::OFF_RED);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);

    const uint32_t warp = warp_id(), lane = lane_id();
    const int h = blockIdx.x / p.nq;
    const int i = blockIdx.x - h * p.nq;
    const bool gather = p.q_rows != nullptr;
    const bool two_pass = p.lse_in == nullptr;
    const int n_iter = p.nk * (two_pass ? 2 : 1);

    if (threadIdx.x == 0) {
        mbar_init(bar(L::B_Q), gather ? 128u : 1u);
        for (int s = 0; s < KST; ++s) { mbar_init(bar(L::B_KF + s), 1); mbar_init(bar(L::B_KE + s), 1); }
        for (int b = 0; b < 2; ++b) { mbar_init(bar(L::B_SF + b), 1); mbar_init(bar(L::B_SE + b), 128); }
        mbar_init(bar(L::B_DRAIN), 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), kEnergyTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const WaitCtl ctl{abort_flag, p.timeout_ns};

    int armed_q = 0, armed_k[KST];
#pragma unroll
    for (int s = 0; s < KST; ++s) armed_k[s] = 0;

    if (warp == 0) {
        if (lane == 0) {
            if (!gather) {
                mbar_arrive_expect_tx(bar(L::B_Q), L::Q_BYTES);
                for (int c = 0; c < CH; ++c)
                    tma_load_3d(smem_u32(sQ + c * kTileM * 128), &tm_q, bar(L::B_Q), c * 64, i * BLK, h);
                armed_q = 1;
            }
            for (int t = 0; t < n_iter; ++t) {
                const int s = t % KST;
                if (!mbar_wait(bar(L::B_KE + s), ((t / KST) & 1) ^ 1, ctl)) break;
                const int j = t % p.nk;
                mbar_arrive_expect_tx(bar(L::B_KF + s), L::K_BYTES);
                for (int c = 0; c < CH; ++c)
                    tma_load_3d(smem_u32(sK + s * L::K_BYTES + c * BLK * 128), &tm_k, bar(L::B_KF + s),
                                c * 64, j * BLK, h);
                ++armed_k[s];
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc_qk = idesc_bf16_f32(kTileM, BLK, false, false);
            const uint32_t sQa = smem_u32(sQ), sKa = smem_u32(sK);
            bool ok = mbar_wait(bar(L::B_Q), 0, ctl);
            for (int t = 0; ok && t < n_iter; ++t) {
                const int s = t % KST, b = t & 1, u = t >> 1;
                if (u >= 1 && !(ok = mbar_wait(bar(L::B_SE + b), (u - 1) & 1, ctl))) break;
                if (!(ok = mbar_wait(bar(L::B_KF + s), (t / KST) & 1, ctl))) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t inner = (kk & 3) * 32;
                    const uint64_t ad = smem_desc_sw128(sQa + (kk >> 2) * kTileM * 128 + inner, 16, 1024);
                    const uint64_t bd =
                        smem_desc_sw128(sKa + s * L::K_BYTES + (kk >> 2) * BLK * 128 + inner, 16, 1024);
                    umma_ss(tmem + b * 128, ad, bd, idesc_qk, kk > 0 ? 1u : 0u);
                }
                umma_commit(bar(L::B_SF + b));
                umma_commit(bar(L::B_KE + s));
            }
        }
    } else {
        const uint32_t q4 = warp & 3;
        const int r = static_cast<int>(q4 * 32 + lane);
        const uint32_t lane_base = (q4 * 32) << 16;
        const int qrow = i * BLK + r;                      // row in the query sequence
        const bool row_ok = r < BLK && qrow < p.Nq;
        if (gather) {
            const __nv_bfloat16* src =
                (qrow < p.Nq) ? p.q + (static_cast<size_t>(h) * p.N + p.q_rows[qrow]) * D : nullptr;
            gather_q_row<D>(sQ, r, src);
            fence_proxy_async_smem();
            mbar_arrive(bar(L::B_Q));
        }
        float m_run = -INFINITY, l_run = 0.f, lse2 = 0.f;
        if (!two_pass && row_ok) lse2 = p.lse_in[static_cast<size_t>(h) * p.Nq + qrow] * 1.4426950408889634f;
        // After a timeout ("dead") a warp keeps iterating without touching tensor memory,
        // so the per-tile named barrier below still sees all 128 threads.
        bool dead = false;
        for (int t = 0; t < n_iter; ++t) {
            const int b = t & 1;
            const int j = t % p.nk;
            const bool pass_lse = two_pass && t < p.nk;
            const int valid = min(BLK, p.N - j * BLK);
            if (!dead) dead = !mbar_wait_warp(bar(L::B_SF + b), (t >> 1) & 1, ctl);
            float s[BLK];
            if (!dead) {
                tc_fence_after();
                uint32_t raw[32];
#pragma unroll
                for (int c = 0; c < BLK / 32; ++c) {
                    tmem_ld32_wait(tmem + lane_base + b * 128 + c * 32, raw);
#pragma unroll
                    for (int e = 0; e < 32; ++e) s[c * 32 + e] = __uint_as_float(raw[e]);
                }
            } else {
#pragma unroll
                for (int c = 0; c < BLK; ++c) s[c] = 0.f;
            }
            tc_fence_before();
            mbar_arrive(bar(L::B_SE + b));          // S buffer may be overwritten now
            if (pass_lse) {
                float mt = -INFINITY;
#pragma unroll
                for (int c = 0; c < BLK; ++c)
                    if (c < valid) mt = fmaxf(mt, s[c]);
                const float m_new = fmaxf(m_run, mt * p.scale_log2);
                float sum = 0.f;
#pragma unroll
                for (int c = 0; c < BLK; ++c)
                    if (c < valid) sum += ex2_approx(fmaf(s[c], p.scale_log2, -m_new));
                l_run = l_run * ex2_approx(m_run - m_new) + sum;
                m_run = m_new;
                if (t == p.nk - 1) lse2 = m_run + lg2_approx(l_run);
            } else {
                float e = 0.f;
                if (row_ok) {
#pragma unroll
                    for (int c = 0; c < BLK; ++c)
                        if (c < valid) e += ex2_approx(fmaf(s[c], p.scale_log2, -lse2));
                }
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) e += __shfl_xor_sync(0xffffffffu, e, off);
                if (lane == 0) red[b * 4 + q4] = e;
                // red[] is double-buffered: a warp reaches the next write to red[b] only
                // after the following tile's barrier, which the reader joins after reading.
                named_bar_sync(1, 128);
                if (warp == 2 && lane == 0 && !dead) {
                    const float tot = ((red[b * 4 + 0] + red[b * 4 + 1]) + red[b * 4 + 2]) + red[b * 4 + 3];
                    float* dst = p.energy + (static_cast<size_t>(h) * p.nq + i) * p.nk + j;
                    *dst = p.accumulate ? *dst + tot : tot;
                }
            }
        }
    }

    __syncthreads();
    if (*abort_flag) {
        constexpr uint64_t kDrainNs = 1000000000ull;
        if (warp == 0 && lane == 0) {
            if (armed_q) mbar_wait_drain(bar(L::B_Q), 0, kDrainNs);
            for (int s = 0; s < KST; ++s)
                if (armed_k[s]) mbar_wait_drain(bar(L::B_KF + s), (armed_k[s] - 1) & 1, kDrainNs);
        }
        if (warp == 1 && lane == 0) {
            umma_commit(bar(L::B_DRAIN));
            mbar_wait_drain(bar(L::B_DRAIN), 0, kDrainNs);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kEnergyTmemCols);
    }
}

}  // namespace calib
