// Fused row-LSE + block-energy pass for sm_100a.
//
// Block energy: split the post-softmax attention matrix P into B x B blocks and sum each
// one (summaries of "Accelerating Text-to-Video Generation with Calibrated Sparse
// Attention": [zh] §2.2A, [de] §2A.1, [pt] §2A.2, [fr] §2.A and §2.B.1).  P is never
// stored:  E[h,i,j] = sum_{r in I_i} sum_{c in J_j} 2^(x_rc - lse2_r),  x = s * scale*log2(e),
// lse2 = LSE / ln 2.
//
// One CTA per (head h, query block i), 320 threads:
//   warp 0      TMA: K_j for every key block, twice when the LSE is not supplied (pass 1
//               computes it, pass 2 sums the blocks).
//   warp 1      TMEM owner (512 columns) and MMA issuer (one elected lane of the converged
//               warp): S = Q K_j^T as a TS MMA, M=128, N=B, K=D.  Q sits in tensor memory
//               as packed bf16 pairs, so only K is read from shared memory (an SS MMA also
//               re-reads Q from shared memory for every key block, and at M=N=128 the
//               operand reads, not the math, set its rate).  S rotates through three
//               buffers; a buffer is handed back as soon as its tile is in registers.
//   warps 2..9  arithmetic, in two groups of four warps (one per TMEM lane quadrant).
//               Group g takes the tiles t with t % 2 == g, every column of each, so the two
//               warps of a sub-partition work on different tiles and one's tensor-memory
//               load and reduction overlap the other's exponentials.  Pass 1: each group
//               keeps an exact running (max, sum) of 2^x over its tiles; the groups are
//               merged once, at the end of the pass, into the row's LSE (kept in a register:
//               the LSE is never written to memory, so no scratch buffer is needed).  Pass 2:
//               each thread sums 2^(x - lse2) over a tile's columns; each warp reduces its 32
//               rows with shuffles, batched over four of its group's key blocks, into a
//               shared-memory table of per-warp partials, and after the last key block the
//               CTA adds the four partials of every block (its group's warps) in a fixed
//               order and writes the row of energies.
// Tensor memory: S buffers at columns [0,128), [128,256), [256,384); Q at [384, 384+D/2).
// [AdaSpa] §2 caches the LSE to reuse it in a later search; a supplied LSE skips pass 1.
#pragma once
#include <cuda_bf16.h>
#include "ptx.cuh"
#include "attn_fwd.cuh"

namespace calib {

constexpr int kEnergyGroups = 2;                          // arithmetic groups (tile parity)
constexpr int kEnergySoftmaxWarps = 4 * kEnergyGroups;    // 8
constexpr int kEnergySoftmaxThreads = 32 * kEnergySoftmaxWarps;
constexpr int kEnergyThreads = 64 + kEnergySoftmaxThreads;
constexpr int kEnergySBufs = 3;
constexpr uint32_t kEnergyTmemCols = 512;
constexpr uint32_t kEnergyTmemQ = 384;
constexpr int kEnergyMaxTokens = 131072;                 // N limit (per-block partial table)
constexpr uint32_t kBarEnergy = 1;                        // named barrier of the arithmetic warps

struct EnergyParams {
    const __nv_bfloat16* q;   // [H, N, D]
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
    static constexpr uint32_t K_BYTES = CH * BLK * 128;
    static constexpr uint32_t OFF_K = 0;
    static constexpr int MAX_NK = kEnergyMaxTokens / BLK;
    static constexpr uint32_t OFF_RED = KST * K_BYTES;    // float [warps][MAX_NK]
    static constexpr uint32_t OFF_XCH = OFF_RED + kEnergySoftmaxWarps * MAX_NK * 4;   // float2 [groups][128]
    static constexpr uint32_t OFF_BAR = OFF_XCH + kEnergyGroups * kTileM * 8;
    static constexpr int B_Q = 0, B_KF = 1, B_KE = B_KF + KST, B_SF = B_KE + KST, B_SE = B_SF + kEnergySBufs,
                         B_DRAIN = B_SE + kEnergySBufs, NBARS = B_DRAIN + 1;
    static constexpr uint32_t OFF_MISC = OFF_BAR + NBARS * 8;   // tmem base, abort flag
    static constexpr uint32_t BYTES = OFF_MISC + 16 + 1024;    // + alignment slack
};

template <int D, int BLK, int KST>
__global__ void __launch_bounds__(kEnergyThreads, 1)
block_energy_kernel(const __grid_constant__ CUtensorMap tm_k, const EnergyParams p) {
    using L = EnergySmem<D, BLK, KST>;
    constexpr int CH = L::CH;
    constexpr int HC = BLK;                               // columns per thread and tile
    constexpr int SB = kEnergySBufs;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    uint8_t* sK = smem + L::OFF_K;
    float* red = reinterpret_cast<float*>(smem + L::OFF_RED);
    float2* xch = reinterpret_cast<float2*>(smem + L::OFF_XCH);
    const uint32_t bar0 = smem_u32(smem + L::OFF_BAR);
    auto bar = [&](int idx) -> uint32_t { return bar0 + 8u * idx; };
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);

    const uint32_t warp = warp_id(), lane = lane_id();
    const int h = blockIdx.x / p.nq;
    const int i = blockIdx.x - h * p.nq;
    const bool two_pass = p.lse_in == nullptr;
    const int nk = p.nk;
    const int n_iter = nk * (two_pass ? 2 : 1);

    if (threadIdx.x == 0) {
        mbar_init(bar(L::B_Q), 128);
        for (int s = 0; s < KST; ++s) { mbar_init(bar(L::B_KF + s), 1); mbar_init(bar(L::B_KE + s), 1); }
        for (int b = 0; b < SB; ++b) {
            mbar_init(bar(L::B_SF + b), 1);
            mbar_init(bar(L::B_SE + b), kEnergySoftmaxThreads / kEnergyGroups);   // one group per tile
        }
        mbar_init(bar(L::B_DRAIN), 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) tma_prefetch_desc(&tm_k);
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), kEnergyTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const WaitCtl ctl{abort_flag, p.timeout_ns};

    int armed_k[KST];
#pragma unroll
    for (int s = 0; s < KST; ++s) armed_k[s] = 0;

    if (warp == 0) {
        // ===================== TMA producer (converged warp, one elected lane issues) ====
        for (int t = 0; t < n_iter; ++t) {
            const int s = t % KST;
            if (!mbar_wait_warp(bar(L::B_KE + s), ((t / KST) & 1) ^ 1, ctl)) break;
            const int j = t < nk ? t : t - nk;
            if (elect_one()) {
                mbar_arrive_expect_tx(bar(L::B_KF + s), L::K_BYTES);
                for (int c = 0; c < CH; ++c)
                    tma_load_3d(smem_u32(sK + s * L::K_BYTES + c * BLK * 128), &tm_k, bar(L::B_KF + s), c * 64,
                                j * BLK, h);
            }
            ++armed_k[s];
        }
    } else if (warp == 1) {
        // ===================== MMA issuer ===============================================
        constexpr uint32_t idesc_qk = idesc_bf16_f32(kTileM, BLK, false, false);
        const uint32_t sKa = smem_u32(sK);
        bool ok = mbar_wait_warp(bar(L::B_Q), 0, ctl);
        for (int t = 0; ok && t < n_iter; ++t) {
            const int s = t % KST, b = t % SB, u = t / SB;
            ok = mbar_wait_warp(bar(L::B_KF + s), (t / KST) & 1, ctl);
            // S buffer b is free once every arithmetic thread has loaded its previous tile
            if (ok && u >= 1) ok = mbar_wait_warp(bar(L::B_SE + b), (u - 1) & 1, ctl);
            if (!ok) break;
            tc_fence_after();
            if (elect_one()) {
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t bd =
                        smem_desc_sw128(sKa + s * L::K_BYTES + (kk >> 2) * BLK * 128 + (kk & 3) * 32, 16, 1024);
                    umma_ts(tmem + b * 128, tmem + kEnergyTmemQ + kk * 8, bd, idesc_qk, kk > 0 ? 1u : 0u);
                }
                umma_commit(bar(L::B_SF + b));
                umma_commit(bar(L::B_KE + s));
            }
        }
    } else {
        // ===================== arithmetic (warps 2..9) ==================================
        const int g = static_cast<int>(warp - 2) >> 2;      // group: tiles of parity g
        const int widx = static_cast<int>(warp) - 2;        // partial-sum table row
        const uint32_t q4 = warp & 3;
        const int r = static_cast<int>(q4 * 32 + lane);     // tile row == TMEM lane
        const uint32_t lane_base = (q4 * 32) << 16;
        const int qrow = i * BLK + r;                       // row in the query sequence
        const bool row_ok = r < BLK && qrow < p.Nq;
        const float sc = p.scale_log2;
        if (g == 0) {
            // Q row -> tensor memory: bf16 pairs in memory order are the packed TS operand
            uint32_t w[32];
            const uint4* src = row_ok ? reinterpret_cast<const uint4*>(
                                            p.q + (static_cast<size_t>(h) * p.N + (p.q_rows ? p.q_rows[qrow] : qrow)) * D)
                                      : nullptr;
#pragma unroll
            for (int c = 0; c < D / 64; ++c) {
#pragma unroll
                for (int v = 0; v < 8; ++v) {
                    const uint4 x = src ? __ldg(src + c * 8 + v) : make_uint4(0, 0, 0, 0);
                    w[4 * v] = x.x;
                    w[4 * v + 1] = x.y;
                    w[4 * v + 2] = x.z;
                    w[4 * v + 3] = x.w;
                }
                tmem_st32(tmem + lane_base + kEnergyTmemQ + c * 32, w);
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar(L::B_Q));
        }

        bool ok = true;
        // Wait for tile t, load this thread's HC columns, hand the S buffer back, mask the
        // columns past N (ragged last key block only).
        auto load_tile = [&](int t, int j, float (&s)[HC]) -> bool {
            const int b = t % SB;
            if (!mbar_wait_warp(bar(L::B_SF + b), (t / SB) & 1, ctl)) return false;
            tc_fence_after();
            {
                uint32_t raw[HC];
                if constexpr (HC == 128) tmem_ld128_wait(tmem + lane_base + b * 128, raw);
                else tmem_ld64_wait(tmem + lane_base + b * 128, raw);
#pragma unroll
                for (int c = 0; c < HC; ++c) s[c] = __uint_as_float(raw[c]);
            }
            tc_fence_before();
            mbar_arrive(bar(L::B_SE + b));
            const int valid = min(BLK, p.N - j * BLK);
            if (valid < HC) {
#pragma unroll
                for (int c = 0; c < HC; ++c)
                    if (c >= valid) s[c] = -INFINITY;
            }
            return true;
        };
        // sum_c 2^(s_c * sc - m) with four independent packed accumulators.  The MUFU exp2
        // unit bounds this pass, so one pair of exponentials in every KP groups of four goes
        // to the FMA pipe (exp2_poly2, relative error below 3e-6): a share of 1/(2 KP).
        // Measured best: 1/4 in pass 1, whose max leaves the FMA pipe less busy, and 1/8 in
        // pass 2 (1/16 and 1/4 there, and 1/2 in pass 1, were slower).  A masked column on
        // the FMA pipe adds about 2^-125 instead of 0, far below any energy's tolerance.
        auto exp_sum = [&](const float (&s)[HC], float m, const int KP) -> float {
            float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
            for (int c = 0; c < HC; c += 4) {
                float x0, x1, x2, x3;
                ffma2(x0, x1, s[c], s[c + 1], sc, sc, -m, -m);
                ffma2(x2, x3, s[c + 2], s[c + 3], sc, sc, -m, -m);
                fadd2(a0, a1, a0, a1, ex2_approx(x0), ex2_approx(x1));
                float y2, y3;
                if ((c / 4) % KP == KP - 1) {
                    exp2_poly2(y2, y3, x2, x3);
                } else {
                    y2 = ex2_approx(x2);
                    y3 = ex2_approx(x3);
                }
                fadd2(a2, a3, a2, a3, y2, y3);
            }
            return (a0 + a1) + (a2 + a3);
        };

        float lse2 = 0.f;
        if (two_pass) {
            // ---- pass 1: exact running (max, sum) of the row over this group's tiles ----
            float m_run = -INFINITY, l_run = 0.f;
            for (int t = g; t < nk; t += kEnergyGroups) {
                float s[HC];
                ok = load_tile(t, t, s);
                if (!ok) break;
                float mx0 = s[0], mx1 = s[1], mx2 = s[2], mx3 = s[3];
#pragma unroll
                for (int c = 4; c + 8 <= HC; c += 8) {
                    mx0 = fmax3(mx0, s[c], s[c + 4]);
                    mx1 = fmax3(mx1, s[c + 1], s[c + 5]);
                    mx2 = fmax3(mx2, s[c + 2], s[c + 6]);
                    mx3 = fmax3(mx3, s[c + 3], s[c + 7]);
                }
                mx0 = fmaxf(mx0, s[HC - 4]);
                mx1 = fmaxf(mx1, s[HC - 3]);
                mx2 = fmaxf(mx2, s[HC - 2]);
                mx3 = fmaxf(mx3, s[HC - 1]);
                const float m_new = fmaxf(m_run, fmax3(mx0, mx1, fmaxf(mx2, mx3)) * sc);
                // a group that has seen only masked columns keeps m = -inf and sum 0
                const float m_sub = m_new == -INFINITY ? 0.f : m_new;
                const float alpha = m_run == -INFINITY ? 0.f : ex2_approx(m_run - m_new);
                l_run = l_run * alpha + exp_sum(s, m_sub, 2);
                m_run = m_new;
            }
            xch[g * kTileM + r] = make_float2(m_run, l_run);
            named_bar_sync(kBarEnergy, kEnergySoftmaxThreads);
            float m = -INFINITY;
#pragma unroll
            for (int gg = 0; gg < kEnergyGroups; ++gg) m = fmaxf(m, xch[gg * kTileM + r].x);
            float lsum = 0.f;
#pragma unroll
            for (int gg = 0; gg < kEnergyGroups; ++gg) {
                const float2 v = xch[gg * kTileM + r];
                if (v.x != -INFINITY) lsum += v.y * ex2_approx(v.x - m);
            }
            lse2 = m + lg2_approx(lsum);
        } else if (row_ok) {
            lse2 = p.lse_in[static_cast<size_t>(h) * p.Nq + qrow] * 1.4426950408889634f;
        }

        // ---- pass 2: block sums of this group's tiles (key block j is tile t0 + j), reduced
        // per warp in batches of four ----
        const int t0 = two_pass ? nk : 0;
        const int jg = (g - t0 % kEnergyGroups + kEnergyGroups) % kEnergyGroups;   // first own block
        for (int jb = jg; ok && jb < nk; jb += 4 * kEnergyGroups) {
            float e4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int j = jb + q * kEnergyGroups;
                if (j < nk && ok) {
                    float s[HC];
                    ok = load_tile(t0 + j, j, s);
                    if (ok && row_ok) e4[q] = exp_sum(s, lse2, 4);
                }
            }
            if (!__all_sync(0xffffffffu, ok)) break;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
#pragma unroll
                for (int q = 0; q < 4; ++q) e4[q] += __shfl_xor_sync(0xffffffffu, e4[q], off);
            }
            if (lane == 0) {
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    if (jb + q * kEnergyGroups < nk) red[widx * L::MAX_NK + jb + q * kEnergyGroups] = e4[q];
            }
        }
        named_bar_sync(kBarEnergy, kEnergySoftmaxThreads);   // every arithmetic warp gets here
        if (!*abort_flag) {
            float* dst = p.energy + (static_cast<size_t>(h) * p.nq + i) * nk;
            for (int j = static_cast<int>(threadIdx.x) - 64; j < nk; j += kEnergySoftmaxThreads) {
                // the partials of block j come from the four warps of the group holding it
                const int w0 = 4 * ((t0 + j) % kEnergyGroups);
                float tot = 0.f;
#pragma unroll
                for (int w = 0; w < 4; ++w) tot += red[(w0 + w) * L::MAX_NK + j];
                dst[j] = p.accumulate ? dst[j] + tot : tot;
            }
        }
    }

    // ---- teardown (also the abort drain) ----------------------------------------
    __syncthreads();
    if (*abort_flag) {
        constexpr uint64_t kDrainNs = 1000000000ull;
        if (warp == 0 && lane == 0) {
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
