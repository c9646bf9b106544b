// Spatial-repetition similarity for sm_100a: for sampled video tokens b, the cosine between
// the post-softmax attention rows of b and of its anchor a(b) = (f, floor(y/s)*s, x).
//
// Calibration marks a (timestep, layer, head) spatially repetitive when the attention
// vectors of different spatial rows of a frame are similar beyond a threshold gamma
// (summaries of "Accelerating Text-to-Video Generation with Calibrated Sparse Attention":
// [zh] §2.2A, [de] §2A.4, [fr] §2.B.3).  P is never stored: per pair,
//   cos = sum_c P_a,c P_b,c / sqrt(sum_c P_a,c^2 * sum_c P_b,c^2),  P_r,c = 2^(x_rc - lse2_r).
//
// One CTA per (head, 64 sampled tokens), 320 threads, the same pipeline as the energy pass:
//   warp 0      TMA: K_j for every key block, twice unless the LSE is supplied.
//   warp 1      TMEM owner and MMA issuer: S = Q K_j^T as a TS MMA (M=128, N=B, K=D) into
//               one of three S buffers, each handed back once loaded.
//   warps 2..9  arithmetic.  Tile row r < 64 is the anchor of sample r, row 64 + r the
//               sample itself (both gathered into tensor memory as Q).  A row is split
//               between two warps by column halves, as in the energy pass.  Pass 1: exact
//               row LSE.  Pass 2: every thread adds its P^2; the sample rows' threads hand
//               their P half-rows, through a double-buffered shared-memory exchange, to the
//               thread of the partner anchor row (same half, same sample), which adds the
//               products.  Each (anchor warp, sample warp) pair has its own full / empty
//               mbarriers per exchange buffer, waited on with the same bounded waits as the
//               rest of the pipeline.  At the end the two halves are added and one thread
//               per sample writes the cosine.
// Tensor memory: S buffers at columns [0,128), [128,256), [256,384); Q at [384, 384+D/2).
#pragma once
#include <cuda_bf16.h>
#include "ptx.cuh"
#include "attn_fwd.cuh"
#include "energy.cuh"

namespace calib {

constexpr int kSimPairs = 64;     // samples per CTA

struct SimParams {
    const __nv_bfloat16* q;   // [H, N, D]
    const int32_t* members;   // [n] sampled video tokens
    const float* lse_in;      // [H, N] natural-log LSE or nullptr
    float* cos_out;           // [H, n]
    int H, N, n, tiles, nk;   // tiles = ceil(n / 64) per head
    int F, Hl, Wl, stride;
    float scale_log2;
    uint64_t timeout_ns;
};

template <int D, int BLK, int KST>
struct SimSmem {
    static constexpr int CH = D / 64;
    static constexpr uint32_t K_BYTES = CH * BLK * 128;
    static constexpr int HC = BLK / 2;
    static constexpr uint32_t OFF_K = 0;
    // sample-row P values handed to the anchor rows: float [2 buffers][2 halves][HC][64],
    // column-major in the sample index so that a warp's stores and loads are contiguous
    static constexpr uint32_t OFF_X = KST * K_BYTES;
    static constexpr uint32_t X_BYTES = 2 * 2 * HC * kSimPairs * 4;
    static constexpr uint32_t OFF_XCH = OFF_X + X_BYTES;            // float2 [2][128] (LSE merge)
    static constexpr uint32_t OFF_FIN = OFF_XCH + 2 * kTileM * 8;    // float [6][64] (final sums)
    static constexpr uint32_t OFF_BAR = OFF_FIN + 6 * kSimPairs * 4;
    // exchange barriers: [full | empty][buffer][warp pair]
    static constexpr int B_Q = 0, B_KF = 1, B_KE = B_KF + KST, B_SF = B_KE + KST, B_SE = B_SF + kEnergySBufs,
                         B_XF = B_SE + kEnergySBufs, B_XE = B_XF + 8, B_DRAIN = B_XE + 8, NBARS = B_DRAIN + 1;
    static constexpr uint32_t OFF_MISC = OFF_BAR + NBARS * 8;
    static constexpr uint32_t BYTES = OFF_MISC + 16 + 1024;
};

// Anchor token of video token t at stride s (text tokens are their own anchor).
__device__ __forceinline__ int sim_anchor(const SimParams& p, int t) {
    const int nv = p.F * p.Hl * p.Wl;
    if (t >= nv) return t;
    const int x = t % p.Wl;
    const int y = (t / p.Wl) % p.Hl;
    const int f = t / (p.Wl * p.Hl);
    return (f * p.Hl + (y / p.stride) * p.stride) * p.Wl + x;
}

template <int D, int BLK, int KST>
__global__ void __launch_bounds__(kEnergyThreads, 1)
repeat_sim_kernel(const __grid_constant__ CUtensorMap tm_k, const SimParams p) {
    using L = SimSmem<D, BLK, KST>;
    constexpr int CH = L::CH;
    constexpr int HC = L::HC;
    constexpr int SB = kEnergySBufs;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    uint8_t* sK = smem + L::OFF_K;
    float* xbuf = reinterpret_cast<float*>(smem + L::OFF_X);
    float2* xch = reinterpret_cast<float2*>(smem + L::OFF_XCH);
    float* fin = reinterpret_cast<float*>(smem + L::OFF_FIN);
    const uint32_t bar0 = smem_u32(smem + L::OFF_BAR);
    auto bar = [&](int idx) -> uint32_t { return bar0 + 8u * idx; };
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);

    const uint32_t warp = warp_id(), lane = lane_id();
    const int h = blockIdx.x / p.tiles;
    const int base = (blockIdx.x - h * p.tiles) * kSimPairs;
    const bool two_pass = p.lse_in == nullptr;
    const int nk = p.nk;
    const int n_iter = nk * (two_pass ? 2 : 1);

    if (threadIdx.x == 0) {
        mbar_init(bar(L::B_Q), 128);
        for (int s = 0; s < KST; ++s) { mbar_init(bar(L::B_KF + s), 1); mbar_init(bar(L::B_KE + s), 1); }
        for (int b = 0; b < SB; ++b) {
            mbar_init(bar(L::B_SF + b), 1);
            mbar_init(bar(L::B_SE + b), kEnergySoftmaxThreads);
        }
        for (int x = 0; x < 8; ++x) { mbar_init(bar(L::B_XF + x), 32); mbar_init(bar(L::B_XE + x), 32); }
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
        // ===================== TMA producer =============================================
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
        const int g = static_cast<int>(warp - 2) >> 2;      // column half
        const uint32_t q4 = warp & 3;
        const int r = static_cast<int>(q4 * 32 + lane);     // tile row == TMEM lane
        const uint32_t lane_base = (q4 * 32) << 16;
        const bool is_anchor = r < kSimPairs;
        const int k = r & (kSimPairs - 1);                  // sample index in this CTA
        const bool pair_ok = base + k < p.n;
        // token of this row: the sample, or its anchor
        int tok = 0;
        if (pair_ok) {
            const int b = p.members[base + k];
            tok = is_anchor ? sim_anchor(p, b) : b;
        }
        const float sc = p.scale_log2;
        if (g == 0) {
            uint32_t w[32];
            const uint4* src =
                pair_ok ? reinterpret_cast<const uint4*>(p.q + (static_cast<size_t>(h) * p.N + tok) * D) : nullptr;
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
        auto load_tile = [&](int t, int j, float (&s)[HC]) -> bool {
            const int b = t % SB;
            if (!mbar_wait_warp(bar(L::B_SF + b), (t / SB) & 1, ctl)) return false;
            tc_fence_after();
            {
                uint32_t raw[HC];
                if constexpr (HC == 64) tmem_ld64_wait(tmem + lane_base + b * 128 + g * HC, raw);
                else tmem_ld32_wait(tmem + lane_base + b * 128 + g * HC, raw);
#pragma unroll
                for (int c = 0; c < HC; ++c) s[c] = __uint_as_float(raw[c]);
            }
            tc_fence_before();
            mbar_arrive(bar(L::B_SE + b));
            const int valid = min(BLK, p.N - j * BLK) - g * HC;
            if (valid < HC) {
#pragma unroll
                for (int c = 0; c < HC; ++c)
                    if (c >= valid) s[c] = -INFINITY;
            }
            return true;
        };

        float lse2 = 0.f;
        if (two_pass) {
            float m_run = -INFINITY, l_run = 0.f;
            for (int t = 0; t < nk; ++t) {
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
                const float m_sub = m_new == -INFINITY ? 0.f : m_new;
                const float alpha = m_run == -INFINITY ? 0.f : ex2_approx(m_run - m_new);
                float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
                for (int c = 0; c < HC; c += 4) {
                    float x0, x1, x2, x3;
                    ffma2(x0, x1, s[c], s[c + 1], sc, sc, -m_sub, -m_sub);
                    ffma2(x2, x3, s[c + 2], s[c + 3], sc, sc, -m_sub, -m_sub);
                    fadd2(a0, a1, a0, a1, ex2_approx(x0), ex2_approx(x1));
                    fadd2(a2, a3, a2, a3, ex2_approx(x2), ex2_approx(x3));
                }
                l_run = l_run * alpha + ((a0 + a1) + (a2 + a3));
                m_run = m_new;
            }
            xch[g * kTileM + r] = make_float2(m_run, l_run);
            named_bar_sync(kBarEnergy, kEnergySoftmaxThreads);
            const float2 v0 = xch[r], v1 = xch[kTileM + r];
            const float m = fmaxf(v0.x, v1.x);
            float lsum = 0.f;
            if (v0.x != -INFINITY) lsum += v0.y * ex2_approx(v0.x - m);
            if (v1.x != -INFINITY) lsum += v1.y * ex2_approx(v1.x - m);
            lse2 = m + lg2_approx(lsum);
        } else if (pair_ok) {
            lse2 = p.lse_in[static_cast<size_t>(h) * p.N + tok] * 1.4426950408889634f;
        }

        // ---- pass 2: squared norms, and the products across each (anchor, sample) pair ----
        // anchor warp (q4 = 0 or 1) and sample warp (q4 + 2) of the same half form one of
        // four warp pairs; buffer b of a pair is full / empty at barriers B_XF / B_XE
        const int wp = 2 * g + (q4 & 1);
        float dot = 0.f, nrm = 0.f;
        const int t0 = two_pass ? nk : 0;
        for (int j = 0; ok && j < nk; ++j) {
            float s[HC];
            ok = load_tile(t0 + j, j, s);
            if (!ok) break;
            float* xb = xbuf + ((j & 1) * 2 + g) * HC * kSimPairs;
            float pv[HC];
            float n0 = 0.f, n1 = 0.f;
#pragma unroll
            for (int c = 0; c < HC; c += 2) {
                float x0, x1;
                ffma2(x0, x1, s[c], s[c + 1], sc, sc, -lse2, -lse2);
                pv[c] = ex2_approx(x0);
                pv[c + 1] = ex2_approx(x1);
                ffma2(n0, n1, pv[c], pv[c + 1], pv[c], pv[c + 1], n0, n1);
            }
            nrm += n0 + n1;
            const int xb_i = (j & 1) * 4 + wp;               // this pair's barrier for buffer j&1
            const uint32_t use = static_cast<uint32_t>(j >> 1);
            if (!is_anchor) {
                // the anchor warp has read this buffer's previous contents
                if (use >= 1) ok = mbar_wait_warp(bar(L::B_XE + xb_i), (use - 1) & 1, ctl);
                if (!ok) break;
#pragma unroll
                for (int c = 0; c < HC; ++c) xb[c * kSimPairs + k] = pv[c];
                mbar_arrive(bar(L::B_XF + xb_i));
            } else {
                ok = mbar_wait_warp(bar(L::B_XF + xb_i), use & 1, ctl);
                if (!ok) break;
                float d0 = 0.f, d1 = 0.f;
#pragma unroll
                for (int c = 0; c < HC; c += 2)
                    ffma2(d0, d1, pv[c], pv[c + 1], xb[c * kSimPairs + k], xb[(c + 1) * kSimPairs + k], d0, d1);
                dot += d0 + d1;
                mbar_arrive(bar(L::B_XE + xb_i));
            }
        }
        // ---- combine the halves: dot and the anchor norm from anchor rows, the sample norm
        // from sample rows; one thread per sample writes the cosine ----
        if (is_anchor) {
            fin[(0 + g) * kSimPairs + k] = dot;
            fin[(2 + g) * kSimPairs + k] = nrm;
        } else {
            fin[(4 + g) * kSimPairs + k] = nrm;
        }
        named_bar_sync(kBarEnergy, kEnergySoftmaxThreads);
        if (is_anchor && g == 0 && pair_ok && !*abort_flag) {
            const float d = fin[k] + fin[kSimPairs + k];
            const float na = fin[2 * kSimPairs + k] + fin[3 * kSimPairs + k];
            const float nb = fin[4 * kSimPairs + k] + fin[5 * kSimPairs + k];
            p.cos_out[static_cast<size_t>(h) * p.n + base + k] = d * rsqrtf(na * nb);
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

// Per head: mean of the cosines over the samples that are not their own anchor, and the
// flag mean > gamma.  One block per head; the fixed-order tree sum makes it deterministic.
__global__ void __launch_bounds__(256)
repeat_flags_kernel(const float* __restrict__ cos, const int32_t* __restrict__ members, int n, int F, int Hl,
                    int Wl, int stride, float gamma, float* __restrict__ mean_out, uint8_t* __restrict__ flag_out) {
    __shared__ float ssum[256];
    __shared__ int scnt[256];
    const int h = blockIdx.x;
    SimParams pp{};
    pp.F = F; pp.Hl = Hl; pp.Wl = Wl; pp.stride = stride;
    float acc = 0.f;
    int cnt = 0;
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
        const int b = members[i];
        if (sim_anchor(pp, b) != b) {
            acc += cos[static_cast<size_t>(h) * n + i];
            ++cnt;
        }
    }
    ssum[threadIdx.x] = acc;
    scnt[threadIdx.x] = cnt;
    __syncthreads();
    for (int off = 128; off > 0; off >>= 1) {
        if (static_cast<int>(threadIdx.x) < off) {
            ssum[threadIdx.x] += ssum[threadIdx.x + off];
            scnt[threadIdx.x] += scnt[threadIdx.x + off];
        }
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        const float mean = scnt[0] > 0 ? ssum[0] / static_cast<float>(scnt[0]) : 0.f;
        mean_out[h] = mean;
        flag_out[h] = mean > gamma ? 1 : 0;
    }
}

}  // namespace calib
