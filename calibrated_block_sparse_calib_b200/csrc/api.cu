// C ABI of libcalibatt.so (declared in include/calibatt.h): argument validation, TMA
// descriptor encoding, and kernel launches.  The library allocates no device memory;
// its only state is the per-device status word in ptx.cuh and a few host-side caches
// (the driver entry point, per-device capability and shared-memory attributes).
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <type_traits>
#include <cstring>
#include <mutex>
#include <set>
#include <utility>
#include <vector>

#include "calibatt.h"
#include "ptx.cuh"
#include "attn_fwd.cuh"
#include "energy.cuh"
#include "select.cuh"
#include "intervals.cuh"
#include "repeat_sim.cuh"

namespace {

constexpr uint64_t kDefaultTimeoutNs = 4000000000ull;   // bounded device waits: 4 s

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
int cdiv(long long a, long long b) { return static_cast<int>((a + b - 1) / b); }

cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

// sm_100 check, cached per device.
calib_status check_device() {
    static std::mutex mu;
    static std::set<int> ok_devices;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return CALIB_ERR_CUDA;
    std::lock_guard<std::mutex> lk(mu);
    if (ok_devices.count(dev)) return CALIB_OK;
    int major = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
        return CALIB_ERR_CUDA;
    if (major != 10) return CALIB_ERR_UNSUPPORTED;
    ok_devices.insert(dev);
    return CALIB_OK;
}

// Raise a kernel's dynamic shared-memory limit once per (kernel, device).
calib_status ensure_smem(const void* fn, int bytes) {
    static std::mutex mu;
    static std::set<std::pair<const void*, int>> done;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return CALIB_ERR_CUDA;
    std::lock_guard<std::mutex> lk(mu);
    if (done.count({fn, dev})) return CALIB_OK;
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
        return CALIB_ERR_CUDA;
    done.insert({fn, dev});
    return CALIB_OK;
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                   CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                   CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// 3-D bf16 view [H][N][D] of a contiguous tensor; box = 64 elements (128 B, the swizzle
// span) x box_rows x 1, 128-byte swizzle, zero fill out of bounds.
bool make_tmap(CUtensorMap* map, const void* base, int D, int N, int H, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(N),
                                static_cast<cuuint64_t>(H)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(N) * D * 2};
    const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

calib_status launch_status() {
    return cudaGetLastError() == cudaSuccess ? CALIB_OK : CALIB_ERR_CUDA;
}

// ---- attention ---------------------------------------------------------------------
// A validated attention call: parameters and tensor maps (K, V, and Q as whole blocks and
// as single rows for gathered anchor rows), launchable in slices of the work list.
struct AttnCall {
    calib::AttnParams p;
    CUtensorMap tk, tv, tq, tq1;
    int D, B, grid;
};

template <int D, int BLK, bool WITH_LSE>
calib_status launch_attn(const AttnCall& c, const calib::AttnParams& p, int grid, cudaStream_t st) {
    constexpr int KST = 3, VST = 2;   // K / V ring depths (with the Q tile, 200 KB at D = B = 128)
    using L = calib::AttnSmem<D, BLK, KST, VST>;
    static_assert(L::BYTES <= 232448, "shared memory budget");
    auto* fn = calib::attn_fwd_kernel<D, BLK, KST, VST, WITH_LSE>;
    if (calib_status s = ensure_smem(reinterpret_cast<const void*>(fn), L::BYTES)) return s;
    fn<<<grid, calib::kAttnThreads, L::BYTES, st>>>(c.tk, c.tv, c.tq, c.tq1, p);
    return launch_status();
}

template <int D, int BLK>
calib_status launch_attn_lse(const AttnCall& c, const calib::AttnParams& p, int grid, cudaStream_t st) {
    return p.lse ? launch_attn<D, BLK, true>(c, p, grid, st) : launch_attn<D, BLK, false>(c, p, grid, st);
}

calib_status attn_prepare(const void* q, const void* k, const void* v, void* o, float* lse, int H, int N,
                          int D, float scale, const calib_block_list* list, const uint32_t* repeat_bits,
                          int F, int Hl, int Wl, int n_text, int stride, uint32_t flags, AttnCall* c) {
    if (!q || !k || !v || !o || !list || !list->row_ptr || !list->col_idx) return CALIB_ERR_INVALID;
    if (flags & ~CALIB_ATTN_OUT_F32) return CALIB_ERR_INVALID;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return CALIB_ERR_INVALID;
    if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return CALIB_ERR_INVALID;
    if (H < 1 || N < 1 || !(scale > 0.f) || !std::isfinite(scale)) return CALIB_ERR_INVALID;
    if (H > 1024 || static_cast<long long>(H) * N * D >= (1ll << 40)) return CALIB_ERR_INVALID;
    const int B = list->block;
    if (B != 64 && B != 128) return CALIB_ERR_INVALID;
    if (D != 64 && D != 128) return CALIB_ERR_UNSUPPORTED;
    const int nb = cdiv(N, B);
    if (list->H != H || list->nq != nb || list->nk != nb || nb > 32767 || H > 32767) return CALIB_ERR_INVALID;
    if (list->work && list->n_work < 0) return CALIB_ERR_INVALID;
    if (calib_status s = check_device()) return s;

    calib::AttnParams& p = c->p;
    p = calib::AttnParams{};
    p.q = static_cast<const __nv_bfloat16*>(q);
    p.o = static_cast<__nv_bfloat16*>(o);
    p.lse = lse;
    p.row_ptr = list->row_ptr;
    p.col_idx = list->col_idx;
    p.work = list->work;
    p.H = H; p.N = N; p.nq = nb; p.nk = nb;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.F = F; p.Hl = Hl; p.Wl = Wl; p.n_text = n_text; p.stride = stride;
    p.Ar = stride > 0 ? (Hl + stride - 1) / stride : 0;
    p.n_anchor = F * p.Ar * Wl + n_text;
    p.nq_anchor = cdiv(p.n_anchor, B);
    for (int w = 0; w < 32; ++w) p.repeat_bits[w] = repeat_bits ? repeat_bits[w] : 0u;
    p.out_f32 = (flags & CALIB_ATTN_OUT_F32) ? 1 : 0;
    p.timeout_ns = kDefaultTimeoutNs;
    c->D = D;
    c->B = B;
    c->grid = list->work ? list->n_work : H * nb;
    if (!make_tmap(&c->tk, k, D, N, H, B) || !make_tmap(&c->tv, v, D, N, H, B) ||
        !make_tmap(&c->tq, q, D, N, H, B) || !make_tmap(&c->tq1, q, D, N, H, 1))
        return CALIB_ERR_CUDA;
    return CALIB_OK;
}

// Launch work items [first, first + count) of a prepared call (items index the work list,
// which must be present unless the slice is the whole grid).
calib_status attn_launch(const AttnCall& c, int first, int count, cudaStream_t st) {
    if (count <= 0) return CALIB_OK;
    calib::AttnParams p = c.p;
    if (p.work) p.work += first;
    else if (first != 0 || count != c.grid) return CALIB_ERR_INVALID;
    if (c.D == 128) return c.B == 128 ? launch_attn_lse<128, 128>(c, p, count, st)
                                      : launch_attn_lse<128, 64>(c, p, count, st);
    return c.B == 128 ? launch_attn_lse<64, 128>(c, p, count, st) : launch_attn_lse<64, 64>(c, p, count, st);
}

calib_status attn_common(const void* q, const void* k, const void* v, void* o, float* lse, int H, int N,
                         int D, float scale, const calib_block_list* list, const uint32_t* repeat_bits,
                         int F, int Hl, int Wl, int n_text, int stride, uint32_t flags, void* stream) {
    AttnCall c;
    if (calib_status s = attn_prepare(q, k, v, o, lse, H, N, D, scale, list, repeat_bits, F, Hl, Wl, n_text,
                                      stride, flags, &c))
        return s;
    return attn_launch(c, 0, c.grid, as_stream(stream));
}

// CUDA events of one call, destroyed on every exit path (a recorded event may be destroyed
// before it completes; its resources are released once it does).
struct EventSet {
    std::vector<cudaEvent_t> ev;
    cudaEvent_t make() {
        cudaEvent_t e = nullptr;
        if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return nullptr;
        ev.push_back(e);
        return e;
    }
    ~EventSet() {
        for (cudaEvent_t e : ev) cudaEventDestroy(e);
    }
};

// Host <-> device transfers of a prepared attention call, overlapped with its kernels per
// chunk of heads (see sparse_attn_fwd_host in calibatt.h).
calib_status host_pipeline(const AttnCall& c, const void* q_host, const void* k_host, const void* v_host,
                           void* o_host, void* q_dev, void* k_dev, void* v_dev, const void* o_dev, int H, int N,
                           int D, const calib_block_list* list, uint32_t flags, int heads_per_chunk,
                           void* stream, void* h2d_stream, void* d2h_stream) {
    const int nb = list->nq;
    // Head chunks need the head-major work order (each head's nq items contiguous, as
    // calib_build_schedule writes it); any other list runs as one chunk.
    const bool chunked = list->work && list->n_work == H * nb && heads_per_chunk < H;
    const int hpc = chunked ? heads_per_chunk : H;
    const size_t in_head = static_cast<size_t>(N) * D * 2;
    const size_t out_head = static_cast<size_t>(N) * D * ((flags & CALIB_ATTN_OUT_F32) ? 4 : 2);
    cudaStream_t st = as_stream(stream);
    cudaStream_t sin = h2d_stream ? as_stream(h2d_stream) : st;
    cudaStream_t sout = d2h_stream ? as_stream(d2h_stream) : st;
    EventSet evs;
    cudaEvent_t start = evs.make();
    if (!start || cudaEventRecord(start, st) != cudaSuccess) return CALIB_ERR_CUDA;
    // the copy streams start after the work already queued on the caller's stream
    if (cudaStreamWaitEvent(sin, start, 0) != cudaSuccess || cudaStreamWaitEvent(sout, start, 0) != cudaSuccess)
        return CALIB_ERR_CUDA;
    // The step ends with the last chunk's kernel and copy-back after the last host-to-device
    // copy, so when there are several chunks the last chunk's heads go one per chunk.
    for (int h0 = 0, h1 = 0; h0 < H; h0 = h1) {
        h1 = h0 + hpc < H ? h0 + hpc : H;
        if (h1 == H && h0 > 0) h1 = h0 + 1;
        const size_t off = static_cast<size_t>(h0) * in_head, len = static_cast<size_t>(h1 - h0) * in_head;
        // one copy per tensor and chunk
        if (cudaMemcpyAsync(static_cast<char*>(q_dev) + off, static_cast<const char*>(q_host) + off, len,
                            cudaMemcpyHostToDevice, sin) != cudaSuccess ||
            cudaMemcpyAsync(static_cast<char*>(k_dev) + off, static_cast<const char*>(k_host) + off, len,
                            cudaMemcpyHostToDevice, sin) != cudaSuccess ||
            cudaMemcpyAsync(static_cast<char*>(v_dev) + off, static_cast<const char*>(v_host) + off, len,
                            cudaMemcpyHostToDevice, sin) != cudaSuccess)
            return CALIB_ERR_CUDA;
        cudaEvent_t in_ready = evs.make();
        if (!in_ready || cudaEventRecord(in_ready, sin) != cudaSuccess ||
            cudaStreamWaitEvent(st, in_ready, 0) != cudaSuccess)
            return CALIB_ERR_CUDA;
        const int first = chunked ? h0 * nb : 0, count = chunked ? (h1 - h0) * nb : c.grid;
        if (calib_status s = attn_launch(c, first, count, st)) return s;
        cudaEvent_t out_ready = evs.make();
        if (!out_ready || cudaEventRecord(out_ready, st) != cudaSuccess ||
            cudaStreamWaitEvent(sout, out_ready, 0) != cudaSuccess)
            return CALIB_ERR_CUDA;
        const size_t ooff = static_cast<size_t>(h0) * out_head, olen = static_cast<size_t>(h1 - h0) * out_head;
        if (cudaMemcpyAsync(static_cast<char*>(o_host) + ooff, static_cast<const char*>(o_dev) + ooff, olen,
                            cudaMemcpyDeviceToHost, sout) != cudaSuccess)
            return CALIB_ERR_CUDA;
    }
    // the caller's stream is ordered after the last copy of O
    cudaEvent_t done = evs.make();
    if (!done || cudaEventRecord(done, sout) != cudaSuccess || cudaStreamWaitEvent(st, done, 0) != cudaSuccess)
        return CALIB_ERR_CUDA;
    return CALIB_OK;
}

// Validated repeat geometry: token count N = F*Hl*Wl + n_text and the head bit set.
calib_status repeat_geometry(int H, int F, int Hl, int Wl, int n_text, int stride, const uint8_t* head_repeat,
                             uint32_t* bits, int* N_out) {
    if (!head_repeat || calib_anchor_count(F, Hl, Wl, n_text, stride) < 0 || H < 1 || H > 1024)
        return CALIB_ERR_INVALID;
    const long long N = static_cast<long long>(F) * Hl * Wl + n_text;
    if (N > (1ll << 31) - 1) return CALIB_ERR_INVALID;
    for (int w = 0; w < 32; ++w) bits[w] = 0u;
    for (int h = 0; h < H; ++h)
        if (head_repeat[h]) bits[h >> 5] |= 1u << (h & 31);
    *N_out = static_cast<int>(N);
    return CALIB_OK;
}

// ---- energy ------------------------------------------------------------------------
template <int D, int BLK>
calib_status launch_energy(const CUtensorMap& tk, const calib::EnergyParams& p, int grid, cudaStream_t st) {
    constexpr int KST = 4;
    using L = calib::EnergySmem<D, BLK, KST>;
    static_assert(L::BYTES <= 232448, "shared memory budget");
    auto* fn = calib::block_energy_kernel<D, BLK, KST>;
    if (calib_status s = ensure_smem(reinterpret_cast<const void*>(fn), L::BYTES)) return s;
    fn<<<grid, calib::kEnergyThreads, L::BYTES, st>>>(tk, p);
    return launch_status();
}

// ---- spatial-repetition similarity -----------------------------------------------------
template <int D, int BLK>
calib_status launch_sim(const CUtensorMap& tk, const calib::SimParams& p, int grid, cudaStream_t st) {
    constexpr int KST = 4;
    using L = calib::SimSmem<D, BLK, KST>;
    static_assert(L::BYTES <= 232448, "shared memory budget");
    auto* fn = calib::repeat_sim_kernel<D, BLK, KST>;
    if (calib_status s = ensure_smem(reinterpret_cast<const void*>(fn), L::BYTES)) return s;
    fn<<<grid, calib::kEnergyThreads, L::BYTES, st>>>(tk, p);
    return launch_status();
}

int rows_grid(long long rows) { return static_cast<int>((rows + 3) / 4); }   // 4 warps per block

}  // namespace

extern "C" {

const char* calib_status_string(calib_status s) {
    switch (s) {
        case CALIB_OK: return "CALIB_OK";
        case CALIB_ERR_INVALID: return "CALIB_ERR_INVALID";
        case CALIB_ERR_UNSUPPORTED: return "CALIB_ERR_UNSUPPORTED";
        case CALIB_ERR_CUDA: return "CALIB_ERR_CUDA";
        case CALIB_ERR_TIMEOUT: return "CALIB_ERR_TIMEOUT";
    }
    return "CALIB_ERR_UNKNOWN";
}

calib_status calib_device_check(void* stream) {
    if (cudaStreamSynchronize(as_stream(stream)) != cudaSuccess) return CALIB_ERR_CUDA;
    uint32_t v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, calib::g_status, sizeof(v)) != cudaSuccess) return CALIB_ERR_CUDA;
    if (v && cudaMemcpyToSymbol(calib::g_status, &zero, sizeof(zero)) != cudaSuccess) return CALIB_ERR_CUDA;
    if (v & calib::STATUS_TIMEOUT) return CALIB_ERR_TIMEOUT;
    if (v & (calib::STATUS_BAD_ENERGY | calib::STATUS_BAD_LIST)) return CALIB_ERR_INVALID;
    return CALIB_OK;
}

calib_status calib_block_energy(const void* q, const void* k, const float* lse, int H, int N, int D, int block,
                                float scale, const int32_t* q_rows, int n_q, float* energy, int accumulate,
                                void* stream) {
    if (!q || !k || !energy || !aligned16(q) || !aligned16(k)) return CALIB_ERR_INVALID;
    if ((reinterpret_cast<uintptr_t>(energy) & 3u) || (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)))
        return CALIB_ERR_INVALID;
    if (H < 1 || N < 1 || !(scale > 0.f) || !std::isfinite(scale)) return CALIB_ERR_INVALID;
    if (block != 64 && block != 128) return CALIB_ERR_INVALID;
    if (D != 64 && D != 128) return CALIB_ERR_UNSUPPORTED;
    const int Nq = q_rows ? n_q : N;
    if (q_rows && n_q < 1) return CALIB_ERR_INVALID;
    const int nq = cdiv(Nq, block), nk = cdiv(N, block);
    if (static_cast<long long>(H) * nq > (1ll << 31) - 1) return CALIB_ERR_INVALID;
    if (N > calib::kEnergyMaxTokens) return CALIB_ERR_UNSUPPORTED;
    if (calib_status s = check_device()) return s;
    calib::EnergyParams p{};
    p.q = static_cast<const __nv_bfloat16*>(q);
    p.q_rows = q_rows;
    p.lse_in = lse;
    p.energy = energy;
    p.H = H; p.N = N; p.Nq = Nq; p.nq = nq; p.nk = nk;
    p.accumulate = accumulate ? 1 : 0;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.timeout_ns = kDefaultTimeoutNs;
    CUtensorMap tk;
    if (!make_tmap(&tk, k, D, N, H, block)) return CALIB_ERR_CUDA;
    cudaStream_t st = as_stream(stream);
    const int grid = H * nq;
    if (D == 128) return block == 128 ? launch_energy<128, 128>(tk, p, grid, st) : launch_energy<128, 64>(tk, p, grid, st);
    return block == 128 ? launch_energy<64, 128>(tk, p, grid, st) : launch_energy<64, 64>(tk, p, grid, st);
}

calib_status calib_select_mask_batched(const float* energy, int nb, int H, int nq, int nk, const double* tau,
                                       const uint8_t* force_keep, uint8_t* mask_out, int32_t* count_accum,
                                       void* stream) {
    if (!energy || !tau || (!mask_out && !count_accum)) return CALIB_ERR_INVALID;
    if (nb < 1 || nb > calib::kSelMaxBatch || H < 1 || nq < 1 || nk < 1) return CALIB_ERR_INVALID;
    if (nk > 32 * calib::kSelMaxPerLane) return CALIB_ERR_UNSUPPORTED;
    if ((reinterpret_cast<uintptr_t>(energy) & 3u) || (reinterpret_cast<uintptr_t>(count_accum) & 3u))
        return CALIB_ERR_INVALID;
    if (static_cast<long long>(nb) * H * nq * nk > (1ll << 31) - 1) return CALIB_ERR_INVALID;
    for (int b = 0; b < nb; ++b)
        if (!(tau[b] > 0.0) || !(tau[b] <= 1.0)) return CALIB_ERR_INVALID;
    if (calib_status s = check_device()) return s;
    calib::SelectParams p{};
    p.energy = energy;
    p.force = force_keep;
    p.mask_out = mask_out;
    p.count_accum = count_accum;
    p.nb = nb; p.rows = H * nq; p.nq = nq; p.nk = nk;
    for (int b = 0; b < nb; ++b) p.tau[b] = tau[b];
    // one warp per (row, chunk of entries): enough warps to fill every SM a few times over,
    // and each warp walks its chunk of entries so that vote counts accumulate in registers
    const long long target = 148ll * 48;
    int n_chunks = static_cast<int>(std::min<long long>(nb, std::max<long long>(1, (target + p.rows - 1) / p.rows)));
    p.chunk = (nb + n_chunks - 1) / n_chunks;
    p.n_chunks = (nb + p.chunk - 1) / p.chunk;
    p.vec = ((nk & 3) == 0 && (reinterpret_cast<uintptr_t>(energy) & 15u) == 0 &&
             (!mask_out || (reinterpret_cast<uintptr_t>(mask_out) & 3u) == 0)) ? 1 : 0;
    const long long warps = static_cast<long long>(p.rows) * p.n_chunks;
    const int grid = static_cast<int>((warps + calib::kSelWarps - 1) / calib::kSelWarps);
    cudaStream_t st = as_stream(stream);
    // energies per lane: the smallest instantiated count covering the row
    auto launch = [&](auto mpl) {
        calib::select_mask_kernel<decltype(mpl)::value><<<grid, calib::kSelWarps * 32, 0, st>>>(p);
    };
    if (nk <= 64) launch(std::integral_constant<int, 2>{});
    else if (nk <= 128) launch(std::integral_constant<int, 4>{});
    else if (nk <= 256) launch(std::integral_constant<int, 8>{});
    else if (nk <= 512) launch(std::integral_constant<int, 16>{});
    else if (nk <= 640) launch(std::integral_constant<int, 20>{});
    else launch(std::integral_constant<int, 32>{});
    return launch_status();
}

calib_status calib_select_mask(const float* energy, int H, int nq, int nk, double tau, const uint8_t* force_keep,
                               uint8_t* mask_out, int32_t* count_accum, void* stream) {
    if (!mask_out) return CALIB_ERR_INVALID;
    return calib_select_mask_batched(energy, 1, H, nq, nk, &tau, force_keep, mask_out, count_accum, stream);
}

calib_status calib_energy_mean(const float* energy_sum, int64_t count, int n_inputs, float* mean_out,
                               void* stream) {
    if (!energy_sum || !mean_out || count < 1 || n_inputs < 1 || n_inputs > (1 << 24)) return CALIB_ERR_INVALID;
    if ((reinterpret_cast<uintptr_t>(energy_sum) & 3u) || (reinterpret_cast<uintptr_t>(mean_out) & 3u))
        return CALIB_ERR_INVALID;
    if (calib_status s = check_device()) return s;
    const long long want = (count / 4 + 255) / 256;
    const int grid = static_cast<int>(std::max<long long>(1, std::min<long long>(want, 148ll * 8)));
    calib::energy_mean_kernel<<<grid, 256, 0, as_stream(stream)>>>(energy_sum, count, static_cast<float>(n_inputs),
                                                                   mean_out);
    return launch_status();
}

calib_status calib_aggregate_masks(const int32_t* counts, int H, int nq, int nk, int n_inputs, int rho_num,
                                   int rho_den, uint8_t* mask_out, void* stream) {
    if (!counts || !mask_out) return CALIB_ERR_INVALID;
    if (H < 1 || nq < 1 || nk < 1 || n_inputs < 1 || rho_num < 0 || rho_den < 1 || rho_num > rho_den)
        return CALIB_ERR_INVALID;
    if (static_cast<long long>(H) * nq * nk > (1ll << 31) - 1) return CALIB_ERR_INVALID;
    if (calib_status s = check_device()) return s;
    const int rows = H * nq;
    calib::aggregate_kernel<<<rows_grid(rows), 128, 0, as_stream(stream)>>>(counts, rows, nk, n_inputs, rho_num,
                                                                             rho_den, mask_out);
    return launch_status();
}

calib_status calib_mask_to_csr(const uint8_t* mask, int H, int nq, int nk, int32_t* row_ptr_out,
                               int16_t* col_idx_out, void* stream) {
    if (!mask || !row_ptr_out || !col_idx_out) return CALIB_ERR_INVALID;
    if (H < 1 || nq < 1 || nk < 1 || nk > 32767) return CALIB_ERR_INVALID;
    if (static_cast<long long>(H) * nq * nk > (1ll << 31) - 1) return CALIB_ERR_INVALID;
    if (calib_status s = check_device()) return s;
    const int rows = H * nq;
    cudaStream_t st = as_stream(stream);
    calib::csr_count_kernel<<<rows_grid(rows), 128, 0, st>>>(mask, rows, nk, row_ptr_out);
    calib::csr_scan_kernel<<<1, 1024, 0, st>>>(row_ptr_out, rows);
    calib::csr_fill_kernel<<<rows_grid(rows), 128, 0, st>>>(mask, rows, nk, row_ptr_out, col_idx_out);
    return launch_status();
}

calib_status calib_csr_to_intervals(const int32_t* row_ptr, const int16_t* col_idx, int H, int nq,
                                    int32_t* iv_ptr_out, int16_t* iv_start_out, int16_t* iv_len_out, void* stream) {
    if (!row_ptr || !col_idx || !iv_ptr_out || !iv_start_out || !iv_len_out) return CALIB_ERR_INVALID;
    if (H < 1 || nq < 1 || static_cast<long long>(H) * nq > (1ll << 31) - 2) return CALIB_ERR_INVALID;
    if (calib_status s = check_device()) return s;
    const int rows = H * nq;
    cudaStream_t st = as_stream(stream);
    calib::iv_count_kernel<<<rows_grid(rows), 128, 0, st>>>(row_ptr, col_idx, rows, iv_ptr_out);
    calib::csr_scan_kernel<<<1, 1024, 0, st>>>(iv_ptr_out, rows);
    calib::iv_fill_kernel<<<rows_grid(rows), 128, 0, st>>>(row_ptr, col_idx, rows, iv_ptr_out, iv_start_out,
                                                           iv_len_out);
    return launch_status();
}

calib_status calib_intervals_to_csr(const int32_t* iv_ptr, const int16_t* iv_start, const int16_t* iv_len, int H,
                                    int nq, int32_t* row_ptr_out, int16_t* col_idx_out, void* stream) {
    if (!iv_ptr || !iv_start || !iv_len || !row_ptr_out) return CALIB_ERR_INVALID;
    if (H < 1 || nq < 1 || static_cast<long long>(H) * nq > (1ll << 31) - 2) return CALIB_ERR_INVALID;
    if (calib_status s = check_device()) return s;
    const int rows = H * nq;
    cudaStream_t st = as_stream(stream);
    calib::iv_total_kernel<<<rows_grid(rows), 128, 0, st>>>(iv_ptr, iv_len, rows, row_ptr_out);
    calib::csr_scan_kernel<<<1, 1024, 0, st>>>(row_ptr_out, rows);
    if (col_idx_out)
        calib::iv_expand_kernel<<<rows_grid(rows), 128, 0, st>>>(iv_ptr, iv_start, iv_len, rows, row_ptr_out,
                                                                 col_idx_out);
    return launch_status();
}

calib_status calib_repeat_similarity(const void* q, const void* k, const float* lse, int H, int N, int D, int block,
                                     float scale, int F, int Hl, int Wl, int stride, const int32_t* members, int n,
                                     float* cos_out, void* stream) {
    if (!q || !k || !members || !cos_out || !aligned16(q) || !aligned16(k)) return CALIB_ERR_INVALID;
    if ((reinterpret_cast<uintptr_t>(cos_out) & 3u) || (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)))
        return CALIB_ERR_INVALID;
    if (H < 1 || N < 1 || n < 1 || !(scale > 0.f) || !std::isfinite(scale)) return CALIB_ERR_INVALID;
    if (F < 1 || Hl < 1 || Wl < 1 || stride < 1 || static_cast<long long>(F) * Hl * Wl > N) return CALIB_ERR_INVALID;
    if (block != 64 && block != 128) return CALIB_ERR_INVALID;
    if (D != 64 && D != 128) return CALIB_ERR_UNSUPPORTED;
    const int tiles = cdiv(n, calib::kSimPairs);
    if (static_cast<long long>(H) * tiles > (1ll << 31) - 1) return CALIB_ERR_INVALID;
    if (calib_status s = check_device()) return s;
    calib::SimParams p{};
    p.q = static_cast<const __nv_bfloat16*>(q);
    p.members = members;
    p.lse_in = lse;
    p.cos_out = cos_out;
    p.H = H; p.N = N; p.n = n; p.tiles = tiles; p.nk = cdiv(N, block);
    p.F = F; p.Hl = Hl; p.Wl = Wl; p.stride = stride;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.timeout_ns = kDefaultTimeoutNs;
    CUtensorMap tk;
    if (!make_tmap(&tk, k, D, N, H, block)) return CALIB_ERR_CUDA;
    cudaStream_t st = as_stream(stream);
    const int grid = H * tiles;
    if (D == 128) return block == 128 ? launch_sim<128, 128>(tk, p, grid, st) : launch_sim<128, 64>(tk, p, grid, st);
    return block == 128 ? launch_sim<64, 128>(tk, p, grid, st) : launch_sim<64, 64>(tk, p, grid, st);
}

calib_status calib_repeat_flags(const float* cos, const int32_t* members, int H, int n, int F, int Hl, int Wl,
                                int stride, float gamma, float* mean_out, uint8_t* flag_out, void* stream) {
    if (!cos || !members || !mean_out || !flag_out) return CALIB_ERR_INVALID;
    if (H < 1 || n < 1 || F < 1 || Hl < 1 || Wl < 1 || stride < 1 || !std::isfinite(gamma)) return CALIB_ERR_INVALID;
    if (calib_status s = check_device()) return s;
    calib::repeat_flags_kernel<<<H, 256, 0, as_stream(stream)>>>(cos, members, n, F, Hl, Wl, stride, gamma, mean_out,
                                                                  flag_out);
    return launch_status();
}

calib_status calib_build_schedule(const int32_t* row_ptr, int H, int nq, int32_t* work_out, void* stream) {
    if (!row_ptr || !work_out) return CALIB_ERR_INVALID;
    if (H < 1 || nq < 1 || H > 32767 || nq > 65535) return CALIB_ERR_INVALID;
    if (calib_status s = check_device()) return s;
    const int bytes = calib::kSchedBins * 4;
    if (calib_status s = ensure_smem(reinterpret_cast<const void*>(calib::schedule_kernel), bytes)) return s;
    calib::schedule_kernel<<<H, 1024, bytes, as_stream(stream)>>>(row_ptr, nq, work_out);
    return launch_status();
}

int64_t calib_anchor_count(int F, int Hl, int Wl, int n_text, int stride) {
    if (F < 1 || Hl < 1 || Wl < 1 || n_text < 0 || stride < 1) return -1;
    const int64_t Ar = (Hl + stride - 1) / stride;
    return static_cast<int64_t>(F) * Ar * Wl + n_text;
}

calib_status calib_anchor_rows(int F, int Hl, int Wl, int n_text, int stride, int32_t* rows_out, void* stream) {
    const int64_t na = calib_anchor_count(F, Hl, Wl, n_text, stride);
    if (!rows_out || na < 0 || static_cast<int64_t>(F) * Hl * Wl + n_text > (1ll << 31) - 1) return CALIB_ERR_INVALID;
    if (calib_status s = check_device()) return s;
    const int Ar = (Hl + stride - 1) / stride;
    const int n = static_cast<int>(na);
    calib::anchor_rows_kernel<<<cdiv(n, 256), 256, 0, as_stream(stream)>>>(F, Hl, Wl, n_text, stride, Ar, n,
                                                                            rows_out);
    return launch_status();
}

calib_status sparse_attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse_opt, int H, int N,
                             int D, float scale, const calib_block_list* list, uint32_t flags, void* stream) {
    return attn_common(q, k, v, o, lse_opt, H, N, D, scale, list, nullptr, 1, 1, N, 0, 1, flags, stream);
}

calib_status sparse_attn_fwd_host(const void* q_host, const void* k_host, const void* v_host, void* o_host,
                                  void* q_dev, void* k_dev, void* v_dev, void* o_dev, float* lse_opt, int H,
                                  int N, int D, float scale, const calib_block_list* list, uint32_t flags,
                                  int heads_per_chunk, void* stream, void* h2d_stream, void* d2h_stream) {
    if (!q_host || !k_host || !v_host || !o_host || heads_per_chunk < 1) return CALIB_ERR_INVALID;
    AttnCall c;
    if (calib_status s = attn_prepare(q_dev, k_dev, v_dev, o_dev, lse_opt, H, N, D, scale, list, nullptr, 1, 1, N,
                                      0, 1, flags, &c))
        return s;
    return host_pipeline(c, q_host, k_host, v_host, o_host, q_dev, k_dev, v_dev, o_dev, H, N, D, list, flags,
                         heads_per_chunk, stream, h2d_stream, d2h_stream);
}

calib_status sparse_attn_fwd_repeat_host(const void* q_host, const void* k_host, const void* v_host,
                                         void* o_host, void* q_dev, void* k_dev, void* v_dev, void* o_dev,
                                         float* lse_opt, int H, int D, int F, int Hl, int Wl, int n_text,
                                         int stride, const uint8_t* head_repeat, float scale,
                                         const calib_block_list* list, uint32_t flags, int heads_per_chunk,
                                         void* stream, void* h2d_stream, void* d2h_stream) {
    if (!q_host || !k_host || !v_host || !o_host || heads_per_chunk < 1) return CALIB_ERR_INVALID;
    uint32_t bits[32];
    int N = 0;
    if (calib_status s = repeat_geometry(H, F, Hl, Wl, n_text, stride, head_repeat, bits, &N)) return s;
    AttnCall c;
    if (calib_status s = attn_prepare(q_dev, k_dev, v_dev, o_dev, lse_opt, H, N, D, scale, list, bits, F, Hl, Wl,
                                      n_text, stride, flags, &c))
        return s;
    return host_pipeline(c, q_host, k_host, v_host, o_host, q_dev, k_dev, v_dev, o_dev, H, N, D, list, flags,
                         heads_per_chunk, stream, h2d_stream, d2h_stream);
}

calib_status sparse_attn_fwd_repeat(const void* q, const void* k, const void* v, void* o, float* lse_opt, int H,
                                    int D, int F, int Hl, int Wl, int n_text, int stride,
                                    const uint8_t* head_repeat, float scale, const calib_block_list* list,
                                    uint32_t flags, void* stream) {
    uint32_t bits[32];
    int N = 0;
    if (calib_status s = repeat_geometry(H, F, Hl, Wl, n_text, stride, head_repeat, bits, &N)) return s;
    return attn_common(q, k, v, o, lse_opt, H, N, D, scale, list, bits, F, Hl, Wl, n_text, stride, flags, stream);
}

calib_status calib_validate_block_list_host(int H, int nq, int nk, const int32_t* row_ptr, const int16_t* col_idx,
                                            int64_t col_capacity, const int32_t* work, int n_work) {
    if (H < 1 || nq < 1 || nk < 1 || nk > 32767 || !row_ptr || col_capacity < 0) return CALIB_ERR_INVALID;
    const long long rows = static_cast<long long>(H) * nq;
    if (rows > (1ll << 31) - 2 || row_ptr[0] != 0) return CALIB_ERR_INVALID;
    for (long long r = 0; r < rows; ++r) {
        const long long b = row_ptr[r], e = row_ptr[r + 1];
        if (e < b || e - b > nk || e > col_capacity) return CALIB_ERR_INVALID;
        if (e > b && !col_idx) return CALIB_ERR_INVALID;
        for (long long x = b; x < e; ++x) {
            const int j = col_idx[x];
            if (j < 0 || j >= nk || (x > b && j <= col_idx[x - 1])) return CALIB_ERR_INVALID;
        }
    }
    if (work) {
        if (n_work < 0) return CALIB_ERR_INVALID;
        for (int w = 0; w < n_work; ++w) {
            const int32_t item = work[w];
            if (item < 0 || (item >> 16) >= H || (item & 0xFFFF) >= nq) return CALIB_ERR_INVALID;
        }
    }
    return CALIB_OK;
}

calib_status calib_selftest_wait_timeout(uint32_t timeout_us, void* stream) {
    if (calib_status s = check_device()) return s;
    calib::selftest_wait_kernel<<<1, 32, 0, as_stream(stream)>>>(static_cast<uint64_t>(timeout_us) * 1000ull);
    if (cudaGetLastError() != cudaSuccess) return CALIB_ERR_CUDA;
    return calib_device_check(stream);
}

}  // extern "C"
