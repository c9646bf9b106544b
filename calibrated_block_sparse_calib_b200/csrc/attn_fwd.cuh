// Block-sparse attention forward for sm_100a: tcgen05 MMAs accumulating in tensor
// memory, TMA-fed Q/K/V tiles, warp-specialised roles, persistent CTAs fed by cluster
// launch control.
//
// The method computes attention only on the (query block, key block) tiles its
// calibrated skip list keeps, densely inside each tile (summaries of "Accelerating
// Text-to-Video Generation with Calibrated Sparse Attention": [zh] §2.2B, [de] §2B,
// [fr] §2.C), and for spatial-repetition heads only on anchor rows whose output is
// broadcast to the other rows of their frame ([zh] §2.2B, [fr] §2.C).
//
// Work items are (head h, query block i), one per CTA of the grid, in the work list's
// longest-first order.  A CTA that finishes an item takes the next one by cancelling the
// launch of a CTA that has not started yet (clusterlaunchcontrol.try_cancel returns that
// CTA's index), so one CTA per SM runs until the grid is exhausted, items are still
// started in work-list order, and the next item's set-up overlaps the current item:
// its Q tile is loaded, copied into tensor memory and multiplied by its first K tile
// while the current item's last softmax tile and epilogue run.
//
// 352 threads:
//   warp 10     scheduler: obtains the next item (the CTA's own index first, then by
//               cancellation), decodes it (work list, row pointers, the diagonal start of
//               its key list) into a double-buffered item record, and loads its Q tile into
//               shared memory with TMA (one 128-row box, or one box per anchor row of a
//               repeat head; rows past the block or the sequence read as zeros).
//   warp 0      TMA producer: K_j / V_j for each kept j of every item through KST / VST-deep
//               rings shared by consecutive items (K runs one tile ahead of V).
//   warp 1      TMEM owner (512 columns) and MMA issuer (one elected lane of the converged
//               warp): Q copied shared -> tensor memory (tcgen05.cp), then
//               S_t = Q K_j^T           TS MMA, M=128, N=B, K=D: Q from TMEM, K from SMEM;
//               O_h += P_t,h V_j,h      TS MMA, M=128, N=D, K=B/2, for the two column
//                                       halves h of the tile: P from TMEM, V from SMEM.
//               With Q in tensor memory QK reads only K from shared memory (with Q in shared
//               memory too, the operand reads, not the math, set the MMA rate).
//   warps 2..9  softmax + epilogue.  Each query row (TMEM lane) is split between two warps:
//               warps 2..5 own the first half of every key tile's columns, warps 6..9 the
//               second half.  The two halves run INDEPENDENT online-softmax chains (own
//               running max m_h, own row sum l_h, own accumulator O_h), merged once in the
//               epilogue:
//               O = (O_0 2^(m_0-m) + O_1 2^(m_1-m)) / (l_0 2^(m_0-m) + l_1 2^(m_1-m)).
//               Per tile a thread loads its B/2 logits and hands S back at once (so the next
//               QK overlaps this tile's softmax), takes the row max in the log2 domain with
//               lazy rescaling (O_h is rescaled only when m_h grows by more than 2^8),
//               writes P = 2^(x - m_h) as bf16 into the P region once the previous PV has
//               consumed the previous P, and adds the bf16-ROUNDED P into l_h, so the
//               normaliser is exactly the sum of the weights that entered the PV product.
// Each row's key list is walked starting at its diagonal block (the first kept key block
// at or after the query block), where local attention peaks, so the running max is
// usually final after the first tile and O is rarely rescaled.
// Tiles are counted across the CTA's items, so every barrier phase is a global tile (or
// item) count.
// Tensor memory: S = cols [0,128), P = [128,192) (P_0 then P_1, packed bf16 pairs),
// Q = [192, 192+D/2), O_0 = [256, 256+D), O_1 = [256+D, 256+2D).
#pragma once
#include <cuda_bf16.h>
#include "ptx.cuh"

namespace calib {

constexpr int kAttnThreads = 352;
constexpr int kSoftmaxThreads = 256;      // warps 2..9
constexpr int kSchedWarp = 10;
constexpr int kInfoConsumers = 10;        // warps reading each item record: 0..9
constexpr int kTileM = 128;               // query rows per tile (MMA M)
constexpr float kRescaleLog2 = 8.0f;      // rescale O only when the row max grows by > 2^8
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemS = 0;            // S tile (fp32, B columns)
constexpr uint32_t kTmemP = 128;          // P tile (bf16 pairs, B/2 columns: half 0 then half 1)
constexpr uint32_t kTmemQ = 192;          // Q tile (bf16 pairs, D/2 columns)
constexpr uint32_t kTmemO = 256;          // first column of O_0 (O_1 follows at kTmemO + D)

struct AttnParams {
    const __nv_bfloat16* q;   // [H, N, D]
    __nv_bfloat16* o;         // [H, N, D], bf16 (or fp32 when out_f32)
    float* lse;               // [H, N] or nullptr
    const int32_t* row_ptr;   // [H*nq + 1]
    const int16_t* col_idx;
    const int32_t* work;      // [n_items] (h << 16 | i) or nullptr (row order)
    int H, N, nq, nk;
    float scale_log2;         // scale * log2(e)
    // spatial repetition
    int F, Hl, Wl, n_text, stride, Ar, n_anchor, nq_anchor;
    uint32_t repeat_bits[32]; // bit h set: head h is a repeat head
    int out_f32;              // 1: o is fp32 [H, N, D]; 0: bf16
    uint64_t timeout_ns;
};

// One decoded work item, as the scheduler publishes it.
struct ItemInfo {
    int h, i, kbeg, nkept, t0, flags, pad0, pad1;
};
enum : int { ITEM_PROCESS = 0, ITEM_SKIP = 1, ITEM_END = 2 };

// Token index of anchor `a` (compacted order: latent rows 0, s, 2s, ... of each frame,
// every column; then text tokens).
__device__ __forceinline__ int anchor_token(const AttnParams& p, int a) {
    const int per_frame = p.Ar * p.Wl;
    const int nva = p.F * per_frame;
    if (a < nva) {
        const int f = a / per_frame;
        const int rem = a - f * per_frame;
        const int ya = rem / p.Wl;
        const int x = rem - ya * p.Wl;
        return (f * p.Hl + ya * p.stride) * p.Wl + x;
    }
    return p.F * p.Hl * p.Wl + (a - nva);
}

// Write 32 output values of one row (already normalised).
__device__ __forceinline__ void store_row32_bf16(__nv_bfloat16* dst, const uint32_t (&packed)[16]) {
    uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
    for (int v = 0; v < 4; ++v)
        d[v] = make_uint4(packed[4 * v], packed[4 * v + 1], packed[4 * v + 2], packed[4 * v + 3]);
}
__device__ __forceinline__ void store_row32_f32(float* dst, const uint32_t* raw) {
    uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
    for (int v = 0; v < 8; ++v) d[v] = make_uint4(raw[4 * v], raw[4 * v + 1], raw[4 * v + 2], raw[4 * v + 3]);
}

// Cluster launch control: ask to cancel the launch of a CTA that has not started; the
// 16-byte answer lands in shared memory at `resp` and completes `bar` (complete_tx).
__device__ __forceinline__ void clc_try_cancel(uint32_t resp, uint32_t bar) {
    asm volatile("clusterlaunchcontrol.try_cancel.async.shared::cta.mbarrier::complete_tx::bytes.b128 [%0], [%1];"
                 ::"r"(resp), "r"(bar)
                 : "memory");
}
// Decode an answer: true and the cancelled CTA's x index, or false (nothing left to take).
__device__ __forceinline__ bool clc_decode(uint32_t resp, int* x) {
    uint32_t ok, cx;
    asm volatile(
        "{\n\t.reg .pred p;\n\t.reg .b128 r;\n\t"
        "ld.shared.b128 r, [%2];\n\t"
        "clusterlaunchcontrol.query_cancel.is_canceled.pred.b128 p, r;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t"
        "@p clusterlaunchcontrol.query_cancel.get_first_ctaid::x.b32.b128 %1, r;\n\t"
        "@!p mov.u32 %1, 0;\n\t}"
        : "=r"(ok), "=r"(cx)
        : "r"(resp)
        : "memory");
    *x = static_cast<int>(cx);
    return ok != 0;
}
// Copy a 128-row x 32-byte slice of a shared-memory matrix (UMMA descriptor) into tensor
// memory: row r -> lane r, 8 consecutive 32-bit columns from `taddr`.
__device__ __forceinline__ void tmem_cp_128x256b(uint32_t taddr, uint64_t sdesc) {
    asm volatile("tcgen05.cp.cta_group::1.128x256b [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

template <int D, int BLK, int KST, int VST>
struct AttnSmem {
    static constexpr int CH = D / 64;                     // 128-byte chunks per row
    static constexpr uint32_t CHUNK = BLK * 128;          // one 64-column chunk of a K/V tile
    static constexpr uint32_t K_BYTES = CH * CHUNK;
    static constexpr uint32_t QCHUNK = kTileM * 128;      // one 64-column chunk of the Q tile
    static constexpr uint32_t Q_BYTES = CH * QCHUNK;
    static constexpr uint32_t OFF_K = 0;
    static constexpr uint32_t OFF_V = OFF_K + KST * K_BYTES;
    static constexpr uint32_t OFF_Q = OFF_V + VST * K_BYTES;
    // the epilogue's exchange of (m, l) between the two halves of a row, float4 [2][2][128]
    // (double-buffered by item parity)
    static constexpr uint32_t OFF_XCH = OFF_Q + Q_BYTES;
    static constexpr uint32_t OFF_INFO = OFF_XCH + 2 * 2 * kTileM * 16;   // ItemInfo [2]
    static constexpr uint32_t OFF_CLC = OFF_INFO + 2 * sizeof(ItemInfo);   // 16-byte answer
    static constexpr uint32_t OFF_BAR = OFF_CLC + 16;
    // barrier indices
    static constexpr int B_QF = 0, B_QE = 1, B_KF = 2, B_KE = B_KF + KST, B_VF = B_KE + KST,
                         B_VE = B_VF + VST, B_SF = B_VE + VST, B_SE = B_SF + 1, B_PF = B_SE + 1,
                         B_O = B_PF + 1, B_X = B_O + 1, B_IF = B_X + 1, B_IE = B_IF + 2, B_CLC = B_IE + 2,
                         B_DRAIN = B_CLC + 1, NBARS = B_DRAIN + 1;
    static constexpr uint32_t OFF_MISC = OFF_BAR + NBARS * 8;   // tmem base, abort flag
    // + alignment slack; at least 120 KB so that one CTA (holding all 512 TMEM columns)
    // is resident per SM and no CTA waits in tcgen05.alloc.
    static constexpr uint32_t RAW = OFF_MISC + 16 + 1024;
    static constexpr uint32_t BYTES = RAW > 120u * 1024 ? RAW : 120u * 1024;
};

template <int D, int BLK, int KST, int VST, bool WITH_LSE>
__global__ void __launch_bounds__(kAttnThreads, 1)
attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_q1,
                const AttnParams p) {
    using L = AttnSmem<D, BLK, KST, VST>;
    constexpr int CH = L::CH;
    constexpr int HC = BLK / 2;                            // key columns per softmax half
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    uint8_t* sK = smem + L::OFF_K;
    uint8_t* sV = smem + L::OFF_V;
    uint8_t* sQ = smem + L::OFF_Q;
    volatile ItemInfo* info = reinterpret_cast<volatile ItemInfo*>(smem + L::OFF_INFO);
    const uint32_t clc_resp = smem_u32(smem + L::OFF_CLC);
    const uint32_t bar0 = smem_u32(smem + L::OFF_BAR);
    auto bar = [&](int idx) -> uint32_t { return bar0 + 8u * idx; };
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);

    const uint32_t warp = warp_id(), lane = lane_id();

    // ---- setup ------------------------------------------------------------------
    if (threadIdx.x == 0) {
        mbar_init(bar(L::B_QF), 1);
        mbar_init(bar(L::B_QE), 1);
        for (int s = 0; s < KST; ++s) { mbar_init(bar(L::B_KF + s), 1); mbar_init(bar(L::B_KE + s), 1); }
        for (int s = 0; s < VST; ++s) { mbar_init(bar(L::B_VF + s), 1); mbar_init(bar(L::B_VE + s), 1); }
        mbar_init(bar(L::B_SF), 1);
        mbar_init(bar(L::B_SE), kSoftmaxThreads);
        mbar_init(bar(L::B_PF), kSoftmaxThreads);
        mbar_init(bar(L::B_O), 1);
        mbar_init(bar(L::B_X), kSoftmaxThreads);
        for (int s = 0; s < 2; ++s) { mbar_init(bar(L::B_IF + s), 1); mbar_init(bar(L::B_IE + s), kInfoConsumers); }
        mbar_init(bar(L::B_CLC), 1);
        mbar_init(bar(L::B_DRAIN), 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == kSchedWarp && lane == 0) {
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_q1);
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const WaitCtl ctl{abort_flag, p.timeout_ns};

    // Item record n (slot n & 1): wait for it, copy it, release the slot (one arrival per
    // consumer warp).  False on timeout / abort.
    auto read_info = [&](int n, ItemInfo& it) -> bool {
        const int s = n & 1;
        if (!mbar_wait_warp(bar(L::B_IF + s), (n >> 1) & 1, ctl)) return false;
        it.h = info[s].h;
        it.i = info[s].i;
        it.kbeg = info[s].kbeg;
        it.nkept = info[s].nkept;
        it.t0 = info[s].t0;
        it.flags = info[s].flags;
        __syncwarp();
        if (elect_one()) mbar_arrive(bar(L::B_IE + s));
        return true;
    };
    auto is_rep = [&](int h) -> bool { return (p.repeat_bits[h >> 5] >> (h & 31)) & 1u; };
    // list position of step t of an item (rotated to start at the diagonal block)
    auto kidx = [](const ItemInfo& it, int t) -> int {
        const int u = t + it.t0;
        return it.kbeg + (u >= it.nkept ? u - it.nkept : u);
    };

    // bookkeeping for the abort drain
    int armed_k[KST], armed_v[VST];
#pragma unroll
    for (int s = 0; s < KST; ++s) armed_k[s] = 0;
#pragma unroll
    for (int s = 0; s < VST; ++s) armed_v[s] = 0;
    int q_arms = 0;
    bool clc_pending = false;
    int clc_count = 0;

    if (warp == kSchedWarp) {
        // ===================== scheduler (converged warp) ===============================
        int id = static_cast<int>(blockIdx.x);
        for (int n = 0;; ++n) {
            ItemInfo it{0, 0, 0, 0, 0, ITEM_END, 0, 0};
            if (id >= 0) {
                int h, i;
                if (p.work) {
                    const int item = p.work[id];
                    h = item >> 16;
                    i = item & 0xFFFF;
                } else {
                    h = id / p.nq;
                    i = id - h * p.nq;
                }
                it.flags = ITEM_SKIP;
                // an item or row outside the call is skipped and reported
                if (h < 0 || h >= p.H || i >= p.nq) {
                    if (lane == 0) raise_status(STATUS_BAD_LIST);
                } else if (i < (is_rep(h) ? p.nq_anchor : p.nq)) {   // rows past the anchor space: skip
                    const bool rep = is_rep(h);
                    const int lrow = h * p.nq + i;
                    const int kbeg = p.row_ptr[lrow];
                    const int nkept = p.row_ptr[lrow + 1] - kbeg;
                    if (kbeg < 0 || nkept < 0 || nkept > p.nk) {
                        if (lane == 0) raise_status(STATUS_BAD_LIST);
                    } else {
                        // the diagonal block: the first kept key block at or after the key
                        // block holding the query block's first token (the list is ascending,
                        // so one ballot over 32 entries at a time finds it)
                        const int Nq = rep ? p.n_anchor : p.N;
                        const int tok = rep ? anchor_token(p, min(i * BLK, Nq - 1)) : i * BLK;
                        const int jd = tok / BLK;
                        int t0 = 0;
                        for (int b0 = 0; b0 < nkept; b0 += 32) {
                            const int x = b0 + static_cast<int>(lane);
                            const uint32_t ge = __ballot_sync(0xffffffffu, x < nkept && p.col_idx[kbeg + x] >= jd);
                            if (ge) {
                                t0 = b0 + __ffs(ge) - 1;
                                break;
                            }
                        }
                        it = ItemInfo{h, i, kbeg, nkept, t0, ITEM_PROCESS, 0, 0};
                    }
                }
            }
            // publish the record once every consumer has read the one two items back
            const int s = n & 1;
            if (n >= 2 && !mbar_wait_warp(bar(L::B_IE + s), ((n >> 1) - 1) & 1, ctl)) break;
            if (lane == 0) {
                info[s].h = it.h;
                info[s].i = it.i;
                info[s].kbeg = it.kbeg;
                info[s].nkept = it.nkept;
                info[s].t0 = it.t0;
                info[s].flags = it.flags;
                mbar_arrive(bar(L::B_IF + s));
            }
            __syncwarp();
            if (it.flags == ITEM_END) break;
            if (it.flags == ITEM_PROCESS && it.nkept > 0) {
                // Q tile -> shared memory, once the previous one has been copied to TMEM
                if (q_arms > 0 && !mbar_wait_warp(bar(L::B_QE), (q_arms - 1) & 1, ctl)) break;
                const uint32_t qb = bar(L::B_QF);
                if (lane == 0) mbar_arrive_expect_tx(qb, L::Q_BYTES);
                __syncwarp();
                if (!is_rep(it.h)) {
                    if (lane == 0) {
                        for (int c = 0; c < CH; ++c) {
                            tma_load_3d(smem_u32(sQ + c * L::QCHUNK), &tm_q, qb, c * 64, it.i * BLK, it.h);
                            // rows BLK..127 of a 64-row block: a box past the sequence (zeros)
                            if (BLK < kTileM)
                                tma_load_3d(smem_u32(sQ + c * L::QCHUNK + BLK * 128), &tm_q, qb, c * 64, p.N, it.h);
                        }
                    }
                } else {
                    // gathered anchor rows, one box per row; rows past the block or the
                    // anchor sequence read the zero fill past N
                    for (int r = static_cast<int>(lane); r < kTileM; r += 32) {
                        const int a = it.i * BLK + r;
                        const int y = (r < BLK && a < p.n_anchor) ? anchor_token(p, a) : p.N;
                        for (int c = 0; c < CH; ++c)
                            tma_load_3d(smem_u32(sQ + c * L::QCHUNK + r * 128), &tm_q1, qb, c * 64, y, it.h);
                    }
                }
                ++q_arms;
            }
            // the next item: cancel the launch of a CTA that has not started and take its index
            if (lane == 0) {
                mbar_arrive_expect_tx(bar(L::B_CLC), 16);
                clc_try_cancel(clc_resp, bar(L::B_CLC));
            }
            clc_pending = true;
            if (!mbar_wait_warp(bar(L::B_CLC), clc_count & 1, ctl)) break;
            clc_pending = false;
            ++clc_count;
            int x = 0;
            const bool got = clc_decode(clc_resp, &x);
            __syncwarp();
            id = got ? x : -1;
        }
    } else if (warp == 0) {
        // ===================== TMA producer (converged warp, one elected lane issues) ====
        int g = 0;                                            // tiles of earlier items
        for (int n = 0;; ++n) {
            ItemInfo it;
            if (!read_info(n, it)) break;
            if (it.flags == ITEM_END) break;
            if (it.flags != ITEM_PROCESS || it.nkept == 0) continue;
            auto issue_k = [&](int t) -> bool {
                const int u = g + t, s = u % KST;
                if (!mbar_wait_warp(bar(L::B_KE + s), ((u / KST) & 1) ^ 1, ctl)) return false;
                const int j = p.col_idx[kidx(it, t)];
                if (elect_one()) {
                    mbar_arrive_expect_tx(bar(L::B_KF + s), L::K_BYTES);
                    for (int c = 0; c < CH; ++c)
                        tma_load_3d(smem_u32(sK + s * L::K_BYTES + c * L::CHUNK), &tm_k, bar(L::B_KF + s), c * 64,
                                    j * BLK, it.h);
                }
                ++armed_k[s];
                return true;
            };
            auto issue_v = [&](int t) -> bool {
                const int u = g + t, s = u % VST;
                if (!mbar_wait_warp(bar(L::B_VE + s), ((u / VST) & 1) ^ 1, ctl)) return false;
                const int j = p.col_idx[kidx(it, t)];
                if (elect_one()) {
                    mbar_arrive_expect_tx(bar(L::B_VF + s), L::K_BYTES);
                    for (int c = 0; c < CH; ++c)
                        tma_load_3d(smem_u32(sV + s * L::K_BYTES + c * L::CHUNK), &tm_v, bar(L::B_VF + s), c * 64,
                                    j * BLK, it.h);
                }
                ++armed_v[s];
                return true;
            };
            bool ok = issue_k(0);
            for (int t = 0; ok && t < it.nkept; ++t) {
                if (t + 1 < it.nkept) ok = issue_k(t + 1);
                if (ok) ok = issue_v(t);
            }
            if (!ok) break;
            g += it.nkept;
        }
    } else if (warp == 1) {
        // ===================== MMA issuer (converged warp, one elected lane issues) ======
        constexpr uint32_t idesc_qk = idesc_bf16_f32(kTileM, BLK, false, false);
        constexpr uint32_t idesc_pv = idesc_bf16_f32(kTileM, D, false, true);
        const uint32_t sKa = smem_u32(sK), sVa = smem_u32(sV), sQa = smem_u32(sQ);
        // Every tcgen05.mma blocks its issuer while the tensor pipe's short queue is full, so
        // time this warp spends between MMA batches leaves the pipe idle.  Per tile there are
        // two wait points, normally already satisfied when reached: S handed back (and K
        // loaded) before the next QK, and P (and V) before PV.  Each wait's first try_wait is
        // issued before the preceding MMA batch, so its latency overlaps that batch.
        auto qk = [&](int u) {                                // tile u (global count)
            const int s = u % KST;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const uint64_t bd =
                    smem_desc_sw128(sKa + s * L::K_BYTES + (kk >> 2) * L::CHUNK + (kk & 3) * 32, 16, 1024);
                umma_ts(tmem + kTmemS, tmem + kTmemQ + kk * 8, bd, idesc_qk, kk > 0 ? 1u : 0u);
            }
            umma_commit(bar(L::B_SF));
            umma_commit(bar(L::B_KE + s));
        };
        auto pv = [&](int u, bool first) {
            const int sv = u % VST;
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
#pragma unroll
                for (int kk = 0; kk < HC / 16; ++kk) {
                    const uint64_t bd =
                        smem_desc_sw128(sVa + sv * L::K_BYTES + (hf * HC + kk * 16) * 128, L::CHUNK, 1024);
                    umma_ts(tmem + kTmemO + hf * D, tmem + kTmemP + hf * (HC / 2) + kk * 8, bd, idesc_pv,
                            (!first || kk > 0) ? 1u : 0u);
                }
            }
            umma_commit(bar(L::B_O));
            umma_commit(bar(L::B_VE + sv));
        };
        // Q tile of the item starting at tile u: copied from shared memory into the Q columns
        // once the previous item's last QK (tile u - 1) has read them, then QK of tile u once
        // the softmax has loaded S of tile u - 1.
        int qn = 0;                                           // Q tiles copied so far
        auto start_item = [&](int u) -> bool {
            bool ok = mbar_wait_warp(bar(L::B_QF), qn & 1, ctl);
            if (ok && u > 0) ok = mbar_wait_warp(bar(L::B_SF), (u - 1) & 1, ctl);
            if (!ok) return false;
            tc_fence_after();
            if (elect_one()) {
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)
                    tmem_cp_128x256b(tmem + kTmemQ + kk * 8,
                                     smem_desc_sw128(sQa + (kk >> 2) * L::QCHUNK + (kk & 3) * 32, 16, 1024));
                umma_commit(bar(L::B_QE));
            }
            ++qn;
            ok = mbar_wait_warp(bar(L::B_KF + u % KST), (u / KST) & 1, ctl);
            if (ok && u > 0) ok = mbar_wait_warp(bar(L::B_SE), (u - 1) & 1, ctl);
            if (!ok) return false;
            tc_fence_after();
            if (elect_one()) qk(u);
            return true;
        };
        int g = 0;
        ItemInfo cur, nxt;
        bool have_next = false, started = false;
        bool ok = read_info(0, cur);
        for (int n = 0; ok; ++n) {
            if (cur.flags == ITEM_END) break;
            bool next_started = false;
            if (cur.flags == ITEM_PROCESS && cur.nkept > 0) {
                if (!started) ok = start_item(g);
                for (int t = 0; ok && t < cur.nkept; ++t) {
                    const int u = g + t;
                    if (t + 1 < cur.nkept) {
                        // the next QK overwrites S once every softmax thread has loaded S_t
                        const bool tok_s = mbar_test(bar(L::B_SE), u & 1);
                        ok = mbar_wait_warp(bar(L::B_KF + (u + 1) % KST), ((u + 1) / KST) & 1, ctl);
                        if (ok) ok = mbar_wait_warp_tok(bar(L::B_SE), u & 1, tok_s, ctl);
                        if (!ok) break;
                        tc_fence_after();
                        if (elect_one()) qk(u + 1);
                    } else {
                        // last tile: start the next item (Q copy and its first QK) before PV
                        ok = read_info(n + 1, nxt);
                        if (!ok) break;
                        have_next = true;
                        if (nxt.flags == ITEM_PROCESS && nxt.nkept > 0) {
                            ok = start_item(u + 1);
                            if (!ok) break;
                            next_started = true;
                        }
                    }
                    const bool tok_p = mbar_test(bar(L::B_PF), u & 1);
                    ok = mbar_wait_warp(bar(L::B_VF + u % VST), (u / VST) & 1, ctl);
                    if (ok) ok = mbar_wait_warp_tok(bar(L::B_PF), u & 1, tok_p, ctl);
                    if (!ok) break;
                    tc_fence_after();
                    if (elect_one()) pv(u, t == 0);
                }
                g += cur.nkept;
            }
            if (!ok) break;
            if (have_next) {
                cur = nxt;
                have_next = false;
            } else {
                ok = read_info(n + 1, cur);
            }
            started = next_started;
        }
    } else {
        // ===================== softmax + epilogue (warps 2..9) =====================
        const int hf = static_cast<int>(warp - 2) >> 2;    // column half of every key tile
        const uint32_t q4 = warp & 3;
        const int r = static_cast<int>(q4 * 32 + lane);   // tile row == TMEM lane
        const uint32_t lane_base = (q4 * 32) << 16;
        const uint32_t o_col = kTmemO + hf * D;            // this half's accumulator O_h
        const float sc = p.scale_log2;
        int g = 0;
        int nx = 0;                                        // epilogues so far (B_X phases)
        for (int n = 0;; ++n) {
            ItemInfo it;
            if (!read_info(n, it)) break;
            if (it.flags == ITEM_END) break;
            if (it.flags != ITEM_PROCESS) continue;
            const int h = it.h, i = it.i, nkept = it.nkept;
            const bool rep = is_rep(h);
            const int Nq = rep ? p.n_anchor : p.N;
            float m_run = -INFINITY;   // running reference max of this half (log2 domain)
            float l_run = 0.f;         // sum of the bf16-rounded P of this half
            float l_ex = 0.f;          // exact fp32 sum (for the LSE output)
            bool ok = true;
            for (int t = 0; t < nkept; ++t) {
                const int u = g + t;
                const int j = p.col_idx[kidx(it, t)];
                // may be <= 0: the ragged tail, or an index outside the key blocks (masked whole)
                const int valid = (j >= 0 ? min(BLK, p.N - j * BLK) : 0) - hf * HC;
                ok = mbar_wait_warp(bar(L::B_SF), u & 1, ctl);
                if (!ok) break;
                tc_fence_after();
                float s[HC];
                {
                    uint32_t raw[HC];
                    if constexpr (HC == 64) tmem_ld64_wait(tmem + lane_base + kTmemS + hf * HC, raw);
                    else tmem_ld32_wait(tmem + lane_base + kTmemS + hf * HC, raw);
#pragma unroll
                    for (int c = 0; c < HC; ++c) s[c] = __uint_as_float(raw[c]);
                }
                tc_fence_before();
                mbar_arrive(bar(L::B_SE));                 // S may be overwritten by the next QK now
                if (valid < HC) {                          // ragged last key block only
#pragma unroll
                    for (int c = 0; c < HC; ++c)
                        if (c >= valid) s[c] = -INFINITY;
                }
                // row max: four independent three-input chains over s[4 .. HC-5], then the
                // last four columns
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
                const float mt2 = fmax3(mx0, mx1, fmaxf(mx2, mx3)) * sc;
                const bool upd = mt2 > m_run + kRescaleLog2;
                const float m_new = upd ? mt2 : m_run;
                const float alpha = upd ? ex2_approx(m_run - m_new) : 1.f;
                // a half that has seen only masked columns so far keeps m = -inf; its P is 0
                const float m_sub = m_new == -INFINITY ? 0.f : m_new;
                // P = 2^(s*scale_log2 - m): packed FMA, exp2, bf16 pack; the row sum adds the
                // rounded values (unpacked from the bf16 pair).  One exponential pair in 16 is
                // computed on the FMA pipe (exp2_poly2, relative error below 3e-6, far under
                // bf16's spacing): the exponentials of the two warps of a sub-partition are
                // MUFU-bound, and this measured 1-3% faster (1/8: slower than none; 1/32: in
                // between).  A masked column there gives about 2^-125 instead of 0, against a
                // zero-filled V row.
                uint32_t pk[HC / 2];
                float lr0 = 0.f, lr1 = 0.f, lr2 = 0.f, lr3 = 0.f;
                float le0 = 0.f, le1 = 0.f;
#pragma unroll
                for (int c = 0; c < HC; c += 2) {
                    float x0, x1;
                    ffma2(x0, x1, s[c], s[c + 1], sc, sc, -m_sub, -m_sub);
                    float p0, p1;
                    if ((c / 2) % 16 == 15) {
                        exp2_poly2(p0, p1, x0, x1);
                    } else {
                        p0 = ex2_approx(x0);
                        p1 = ex2_approx(x1);
                    }
                    const uint32_t w = pack_bf16x2(p0, p1);
                    pk[c / 2] = w;
                    const float r0 = __uint_as_float(w << 16), r1 = __uint_as_float(w & 0xFFFF0000u);
                    if ((c & 2) == 0) fadd2(lr0, lr1, lr0, lr1, r0, r1);
                    else fadd2(lr2, lr3, lr2, lr3, r0, r1);
                    if constexpr (WITH_LSE) fadd2(le0, le1, le0, le1, p0, p1);
                }
                l_run = l_run * alpha + ((lr0 + lr1) + (lr2 + lr3));
                if constexpr (WITH_LSE) l_ex = l_ex * alpha + (le0 + le1);
                m_run = m_new;
                // The previous P, in the same columns, is the operand of the previous PV; O is
                // rescaled below.  Consume the completion of every PV: an mbarrier parity wait
                // is only unambiguous while the waiter is at most one phase behind, and this
                // item's PV_t cannot start before this P is ready.
                if (t > 0) {
                    ok = mbar_wait_warp(bar(L::B_O), (u - 1) & 1, ctl);
                    if (!ok) break;
                    tc_fence_after();
                }
                const uint32_t p_col = kTmemP + hf * (HC / 2);
                if constexpr (HC == 64) tmem_st32(tmem + lane_base + p_col, *reinterpret_cast<const uint32_t(*)[32]>(pk));
                else tmem_st16(tmem + lane_base + p_col, pk);
                if (__any_sync(0xffffffffu, upd && t > 0)) {
                    // rescale O_h, accumulated through the previous PV, in place
                    const float a_row = (upd && t > 0) ? alpha : 1.f;
                    uint32_t raw[32];
#pragma unroll
                    for (int c = 0; c < D / 32; ++c) {
                        tmem_ld32_wait(tmem + lane_base + o_col + c * 32, raw);
#pragma unroll
                        for (int e = 0; e < 32; ++e) raw[e] = __float_as_uint(__uint_as_float(raw[e]) * a_row);
                        tmem_st32(tmem + lane_base + o_col + c * 32, raw);
                    }
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(bar(L::B_PF));
            }
            // completion of this item's last PV (the loop consumed every earlier one)
            if (ok && nkept > 0) ok = mbar_wait_warp(bar(L::B_O), (g + nkept - 1) & 1, ctl);
            // ---- merge the two halves and write the output ----
            float4* xch = reinterpret_cast<float4*>(smem + L::OFF_XCH) + (nx & 1) * 2 * kTileM;
            xch[hf * kTileM + r] = make_float4(m_run, l_run, l_ex, 0.f);
            mbar_arrive(bar(L::B_X));                      // every softmax thread has written its half
            if (ok) ok = mbar_wait_warp(bar(L::B_X), nx & 1, ctl);
            ++nx;
            tc_fence_after();
            if (!__all_sync(0xffffffffu, ok && !*abort_flag)) break;
            const float4 x0 = xch[r], x1 = xch[kTileM + r];
            const float m = fmaxf(x0.x, x1.x);
            const float w0 = x0.x == -INFINITY ? 0.f : ex2_approx(x0.x - m);
            const float w1 = x1.x == -INFINITY ? 0.f : ex2_approx(x1.x - m);
            const float lsum = x0.y * w0 + x1.y * w1;
            const float inv_l = nkept > 0 ? 1.f / lsum : 0.f;
            const float c0 = w0 * inv_l, c1 = w1 * inv_l;
            float lse_val = -INFINITY;
            if constexpr (WITH_LSE) {
                if (nkept > 0) lse_val = (m + lg2_approx(x0.z * w0 + x1.z * w1)) * 0.69314718055994530942f;
            }
            const bool row_ok = r < BLK && (i * BLK + r) < Nq;
            // destination rows: the row itself, or every token an anchor stands for
            int tok0 = 0, ncopy = 0, copy_stride = 0;
            if (row_ok) {
                const int a = i * BLK + r;
                if (!rep) {
                    tok0 = a;
                    ncopy = 1;
                } else {
                    const int nva = p.F * p.Ar * p.Wl;
                    tok0 = anchor_token(p, a);
                    if (a < nva) {
                        const int ya = (a / p.Wl) % p.Ar;
                        ncopy = min(p.stride, p.Hl - ya * p.stride);
                        copy_stride = p.Wl;
                    } else {
                        ncopy = 1;
                    }
                }
            }
            // this warp writes output columns [hf*D/2, (hf+1)*D/2), reading both halves
#pragma unroll
            for (int cc = 0; cc < D / 64; ++cc) {
                const int c = hf * (D / 64) + cc;             // 32-column chunk index
                uint32_t raw[32];
                if (nkept > 0) {
                    uint32_t raw1[32];
                    tmem_ld32_wait(tmem + lane_base + kTmemO + c * 32, raw);
                    tmem_ld32_wait(tmem + lane_base + kTmemO + D + c * 32, raw1);
#pragma unroll
                    for (int e = 0; e < 32; e += 2) {
                        float y0, y1, z0, z1;
                        ffma2(y0, y1, __uint_as_float(raw1[e]), __uint_as_float(raw1[e + 1]), c1, c1, 0.f, 0.f);
                        ffma2(z0, z1, __uint_as_float(raw[e]), __uint_as_float(raw[e + 1]), c0, c0, y0, y1);
                        raw[e] = __float_as_uint(z0);
                        raw[e + 1] = __float_as_uint(z1);
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e) raw[e] = 0u;
                }
                if (p.out_f32) {
                    for (int cp = 0; cp < ncopy; ++cp) {
                        const size_t tok = static_cast<size_t>(tok0 + cp * copy_stride);
                        store_row32_f32(reinterpret_cast<float*>(p.o) + (static_cast<size_t>(h) * p.N + tok) * D +
                                            c * 32, raw);
                    }
                } else {
                    uint32_t packed[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        packed[e] = pack_bf16x2(__uint_as_float(raw[2 * e]), __uint_as_float(raw[2 * e + 1]));
                    for (int cp = 0; cp < ncopy; ++cp) {
                        const size_t tok = static_cast<size_t>(tok0 + cp * copy_stride);
                        store_row32_bf16(p.o + (static_cast<size_t>(h) * p.N + tok) * D + c * 32, packed);
                    }
                }
            }
            if (p.lse && hf == 0)
                for (int cp = 0; cp < ncopy; ++cp)
                    p.lse[static_cast<size_t>(h) * p.N + tok0 + cp * copy_stride] = lse_val;
            // O is read: the next item's first PV may overwrite it once this thread's P of that
            // item is ready (its PF arrival follows these loads)
            tc_fence_before();
            g += nkept;
        }
    }

    // ---- teardown (also the abort drain) ----------------------------------------
    // After this barrier no role waits any more, so every thread reads the same flag.
    __syncthreads();
    if (*abort_flag) {
        constexpr uint64_t kDrainNs = 1000000000ull;
        if (warp == 0 && lane == 0) {
            for (int s = 0; s < KST; ++s)
                if (armed_k[s]) mbar_wait_drain(bar(L::B_KF + s), (armed_k[s] - 1) & 1, kDrainNs);
            for (int s = 0; s < VST; ++s)
                if (armed_v[s]) mbar_wait_drain(bar(L::B_VF + s), (armed_v[s] - 1) & 1, kDrainNs);
        }
        if (warp == kSchedWarp && lane == 0) {
            if (q_arms) mbar_wait_drain(bar(L::B_QF), (q_arms - 1) & 1, kDrainNs);
            if (clc_pending) mbar_wait_drain(bar(L::B_CLC), clc_count & 1, kDrainNs);
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
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace calib
