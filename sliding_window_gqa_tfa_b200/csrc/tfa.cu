// tfa.cu -- C-ABI boundary of the tiled GQA prefill attention library:
// argument validation, TMA descriptor encoding, launch of the sm_100a kernel,
// the device status word and the host-buffer entry point.
//
// The rejection rules follow tiny-llm "Week 2 Day 5: Tiled Dense Prefill
// Attention", Task 1: BF16 inputs (by the ABI's contract), equal K/V shapes and
// matching batch/head dimensions (one B, Hkv, S for both), Hq % Hkv == 0, and
// the direct operator rejects queries shorter than nine rows.
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <unordered_map>

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include "../../include/tfa.h"
#include "tfa_bwd.cuh"
#include "tfa_kernel.cuh"

namespace {

constexpr int kMaxDevices = 64;

// Scratch of the split schedule, one set per (device, stream) so that calls on
// different streams never share it: a partial slot and a ready flag per
// (CTA, query tile), then two control words (finished launches, finished CTAs).
struct SplitScratch {
    float *partial = nullptr;
    unsigned *ready = nullptr;
    unsigned *ctl = nullptr;
};

// Workspace of the backward pass, per (device, stream), grown on demand: the
// recomputed forward output and per-row log-sum-exp, and delta = rowsum(dO o O).
struct BwdScratch {
    void *o = nullptr;
    float *lse = nullptr, *delta = nullptr;
    size_t rows = 0, o_bytes = 0;
};

constexpr int kVariantsPerD = 18;  // forward kernel variants per head dim (variant_index)
constexpr int kHostStages = 4;     // tfa_prefill_host: most pipeline stages per call (measured best of 4, 8, 16)

struct DeviceState {
    bool init = false;
    int sm_count = 0;
    unsigned *status = nullptr;  // device status word (TFA_DEVICE_TIMEOUT bits)
    bool smem_attr[2 * kVariantsPerD] = {};  // per kernel variant: D, layout, key mask, score mode
    std::unordered_map<cudaStream_t, SplitScratch> split;
    std::unordered_map<cudaStream_t, BwdScratch> bwd;
    bool bwd_attr[4] = {};  // backward kernels prepared, per (D, key mask)
    // staging buffers of tfa_prefill_host, and its copy streams and events
    void *h_buf[5] = {nullptr, nullptr, nullptr, nullptr, nullptr};
    size_t h_cap[5] = {0, 0, 0, 0, 0};
    cudaStream_t h_in = nullptr, h_out = nullptr;
    cudaEvent_t h_ev[2 * kHostStages + 1] = {};
};

std::mutex g_mutex;
DeviceState g_dev[kMaxDevices];
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
thread_local char g_last_error[256] = "";

// Record which CUDA call failed (readable through tfa_last_error) and map it to TFA_ERR_CUDA.
int cuda_fail(const char *what, cudaError_t e) {
    snprintf(g_last_error, sizeof g_last_error, "%s: %s (%d)", what, cudaGetErrorString(e),
             static_cast<int>(e));
    return TFA_ERR_CUDA;
}
int drv_fail(const char *what, int code) {
    snprintf(g_last_error, sizeof g_last_error, "%s: CUresult %d", what, code);
    return TFA_ERR_CUDA;
}

int get_encode_fn() {
    if (g_encode) return TFA_OK;
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
    if (e != cudaSuccess) return cuda_fail("cudaGetDriverEntryPoint", e);
    if (q != cudaDriverEntryPointSuccess || fn == nullptr)
        return drv_fail("cudaGetDriverEntryPoint(cuTensorMapEncodeTiled) query", static_cast<int>(q));
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    return TFA_OK;
}

// Kernel variants per head dim: dense (packed x key mask x score mode: 12),
// ring (packed x plain/softcap: 4) and varlen (plain/softcap: 2); ring and
// varlen take no key mask and write no LSE, varlen is never packed.
constexpr int variant_index(int D, bool km, int mode, int layout, bool pk) {
    const int sc = mode == tfa::kModeSoftcap ? 1 : 0;
    const int v = layout == tfa::kLayoutDense ? (pk ? 6 : 0) + 2 * mode + (km ? 1 : 0)
                  : layout == tfa::kLayoutRing ? 12 + (pk ? 2 : 0) + sc
                                               : 16 + sc;
    return (D == 128 ? kVariantsPerD : 0) + v;
}

// Shared-memory opt-in and the register check for one kernel variant, done
// once per device at first use (never lazily, so a captured call needs neither).
template <int D, bool KM, int MODE, int LY, bool PK>
int prepare_kernel(DeviceState &st) {
    using C = tfa::Cfg<D>;
    auto kern = tfa::tfa_prefill_kernel<D, KM, MODE, LY, PK>;
    // the largest launch of this variant: with a key mask, or a varlen table
    const int smem = KM ? C::kSmemBytesKeyMask : C::kSmemBytesVarlen;
    const int which = variant_index(D, KM, MODE, LY, PK);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return cuda_fail("cudaFuncSetAttribute(max dynamic smem)", e);
    cudaFuncAttributes fa;
    if ((e = cudaFuncGetAttributes(&fa, kern)) != cudaSuccess) return cuda_fail("cudaFuncGetAttributes", e);
    // The setmaxnreg split inside the kernel is sized for exactly kRegsLaunch
    // registers per thread at launch; any other count could leave a warpgroup
    // waiting for registers that do not exist, so refuse to launch.
    if (fa.maxThreadsPerBlock < tfa::kThreads || fa.numRegs != tfa::kRegsLaunch) {
        snprintf(g_last_error, sizeof g_last_error,
                 "kernel uses %d registers/thread (%d expected), at most %d threads fit, %d needed",
                 fa.numRegs, tfa::kRegsLaunch, fa.maxThreadsPerBlock, tfa::kThreads);
        return TFA_ERR_CUDA;
    }
    st.smem_attr[which] = true;
    return TFA_OK;
}

template <int D, bool KM>
int prepare_bwd_kernels(DeviceState &st) {
    const int smem = tfa::bwd::Cfg<D>::kSmemBytes;
    cudaError_t e = cudaFuncSetAttribute(tfa::bwd::dq_kernel<D, KM>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(tfa::bwd::dkv_kernel<D, KM>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return cuda_fail("cudaFuncSetAttribute(backward smem)", e);
    st.bwd_attr[(D == 128 ? 2 : 0) + (KM ? 1 : 0)] = true;
    return TFA_OK;
}

template <int D, bool PK>
int prepare_dense_kernels(DeviceState &st) {
    using namespace tfa;
    int rc = prepare_kernel<D, false, kModePlain, kLayoutDense, PK>(st);
    if (!rc) rc = prepare_kernel<D, true, kModePlain, kLayoutDense, PK>(st);
    if (!rc) rc = prepare_kernel<D, false, kModeSoftcap, kLayoutDense, PK>(st);
    if (!rc) rc = prepare_kernel<D, true, kModeSoftcap, kLayoutDense, PK>(st);
    if (!rc) rc = prepare_kernel<D, false, kModeLse, kLayoutDense, PK>(st);
    if (!rc) rc = prepare_kernel<D, true, kModeLse, kLayoutDense, PK>(st);
    if (!rc) rc = prepare_kernel<D, false, kModePlain, kLayoutRing, PK>(st);
    if (!rc) rc = prepare_kernel<D, false, kModeSoftcap, kLayoutRing, PK>(st);
    return rc;
}

template <int D>
int prepare_forward_kernels(DeviceState &st) {
    using namespace tfa;
    int rc = prepare_dense_kernels<D, false>(st);
    if (!rc) rc = prepare_dense_kernels<D, true>(st);
    if (!rc) rc = prepare_kernel<D, false, kModePlain, kLayoutVarlen, false>(st);
    if (!rc) rc = prepare_kernel<D, false, kModeSoftcap, kLayoutVarlen, false>(st);
    return rc;
}

int prepare_all_kernels(DeviceState &st) {
    int rc = prepare_forward_kernels<64>(st);
    if (!rc) rc = prepare_forward_kernels<128>(st);
    if (!rc) rc = prepare_bwd_kernels<64, false>(st);
    if (!rc) rc = prepare_bwd_kernels<64, true>(st);
    if (!rc) rc = prepare_bwd_kernels<128, false>(st);
    if (!rc) rc = prepare_bwd_kernels<128, true>(st);
    return rc;
}

// First use allocates; that cannot happen inside a CUDA graph capture, so a
// first call made under capture is refused (one ordinary call on the stream
// beforehand creates everything a captured call needs).
int refuse_under_capture(cudaStream_t stream, const char *what) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(stream, &cs) == cudaSuccess && cs == cudaStreamCaptureStatusNone)
        return TFA_OK;
    snprintf(g_last_error, sizeof g_last_error,
             "first use of %s during graph capture: make one call on this stream before capturing it",
             what);
    return TFA_ERR_CAPTURE;
}

// Per-device state, created on first use with that device current.  The
// status word is cleared on `stream` so it is ordered before the first launch.
int device_state(cudaStream_t stream, DeviceState **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail("cudaGetDevice", e);
    if (dev < 0 || dev >= kMaxDevices) return drv_fail("device index out of range", dev);
    DeviceState &st = g_dev[dev];
    if (!st.init) {
        if (int rc = refuse_under_capture(stream, "the device")) return rc;
        if ((e = cudaDeviceGetAttribute(&st.sm_count, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
            return cuda_fail("cudaDeviceGetAttribute", e);
        if ((e = cudaMalloc(&st.status, 256)) != cudaSuccess) return cuda_fail("cudaMalloc(status)", e);
        if ((e = cudaMemsetAsync(st.status, 0, 256, stream)) != cudaSuccess)
            return cuda_fail("cudaMemsetAsync(status)", e);
        if (int rc = get_encode_fn()) return rc;
        if (int rc = prepare_all_kernels(st)) return rc;
        st.init = true;
    }
    *out = &st;
    return TFA_OK;
}

// The split schedule's scratch for `stream`, allocated on first use: 2 slots of
// partial_slot_floats<128> floats and 2 flags per CTA (one CTA per SM at most).
int split_scratch(DeviceState &st, cudaStream_t stream, SplitScratch **out) {
    auto found = st.split.find(stream);
    if (found != st.split.end()) {
        *out = &found->second;
        return TFA_OK;
    }
    if (int rc = refuse_under_capture(stream, "this stream")) return rc;
    SplitScratch ss;
    const size_t slots = 2 * static_cast<size_t>(st.sm_count);
    cudaError_t e = cudaMalloc(&ss.partial, slots * tfa::partial_slot_floats<128>() * sizeof(float));
    if (e != cudaSuccess) return cuda_fail("cudaMalloc(split partials)", e);
    if ((e = cudaMalloc(&ss.ready, (slots + 2) * sizeof(unsigned))) != cudaSuccess) {
        cudaFree(ss.partial);
        return cuda_fail("cudaMalloc(split flags)", e);
    }
    ss.ctl = ss.ready + slots;
    if ((e = cudaMemsetAsync(ss.ready, 0, (slots + 2) * sizeof(unsigned), stream)) != cudaSuccess)
        return cuda_fail("cudaMemsetAsync(split flags)", e);
    *out = &st.split.emplace(stream, ss).first->second;
    return TFA_OK;
}

// The backward workspace for `stream`, at least `rows` rows of D columns.
int bwd_scratch(DeviceState &st, cudaStream_t stream, size_t rows, int D, BwdScratch **out) {
    BwdScratch &bs = st.bwd[stream];
    const size_t o_bytes = rows * static_cast<size_t>(D) * 2;
    if (bs.rows < rows || bs.o_bytes < o_bytes) {
        if (int rc = refuse_under_capture(stream, "a larger backward workspace")) return rc;
        cudaFree(bs.o);
        cudaFree(bs.lse);
        cudaFree(bs.delta);
        bs = BwdScratch{};
        cudaError_t e = cudaMalloc(&bs.o, o_bytes);
        if (e == cudaSuccess) e = cudaMalloc(&bs.lse, rows * sizeof(float));
        if (e == cudaSuccess) e = cudaMalloc(&bs.delta, rows * sizeof(float));
        if (e != cudaSuccess) {
            cudaFree(bs.o);
            cudaFree(bs.lse);
            cudaFree(bs.delta);
            bs = BwdScratch{};
            return cuda_fail("cudaMalloc(backward workspace)", e);
        }
        bs.rows = rows;
        bs.o_bytes = o_bytes;
    }
    *out = &bs;
    return TFA_OK;
}

int validate(const void *q, const void *k, const void *v, const void *o, int B, int Hq, int Hkv,
             int L, int S, int D, float scale, int causal, int window, const float *key_mask,
             bool check_pointers, bool decode = false) {
    if (check_pointers && (!q || !k || !v || !o)) return TFA_ERR_NULL;
    if (Hq < 1 || Hkv < 1 || Hq % Hkv != 0) return TFA_ERR_HEADS;
    if (!decode && L < TFA_MIN_QUERY_ROWS) return TFA_ERR_SHORT_QUERY;
    if (decode && (L < 1 || L > TFA_MAX_DECODE_ROWS)) return TFA_ERR_SHAPE;
    if (B < 1 || S < L) return TFA_ERR_SHAPE;
    // element counts and every index the kernel forms must stay in range
    const long long qrows = static_cast<long long>(B) * Hq * L;
    const long long krows = static_cast<long long>(B) * Hkv * S;
    if (qrows > (1ll << 31) - 1 || krows > (1ll << 31) - 1 || S > (1 << 30)) return TFA_ERR_SHAPE;
    const long long n_items = static_cast<long long>(B) * Hq * ((L + 2 * tfa::kBlockQ - 1) / (2 * tfa::kBlockQ));
    if (n_items > (1ll << 30)) return TFA_ERR_SHAPE;
    if (D != 64 && D != 128) return TFA_ERR_HEAD_DIM;
    if (window > 0 && !causal) return TFA_ERR_WINDOW;
    if (check_pointers) {
        auto mis16 = [](const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) != 0; };
        if (mis16(q) || mis16(k) || mis16(v) || mis16(o)) return TFA_ERR_ALIGN;
        if (key_mask && (reinterpret_cast<uintptr_t>(key_mask) & 3u)) return TFA_ERR_ALIGN;
    }
    if (!std::isfinite(scale)) return TFA_ERR_SCALE;
    return TFA_OK;
}

// 3-D view [planes][rows][D] of a contiguous bf16 tensor, boxes of 128 rows x
// 64 columns (128 bytes) with 128-byte swizzle; rows past the end read as 0.
// token_major: the tensor is [rows][planes][D] (packed variable-length
// layout), viewed with the same [plane][row][D] coordinates.
int encode_map(CUtensorMap *m, const void *ptr, int rows, int planes, int D,
               int box_rows = tfa::kBlockQ, int box_planes = 1, bool token_major = false) {
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows),
                          static_cast<cuuint64_t>(planes)};
    const cuuint64_t row_bytes = static_cast<cuuint64_t>(D) * 2;
    cuuint64_t strides[2] = {token_major ? row_bytes * static_cast<cuuint64_t>(planes) : row_bytes,
                             token_major ? row_bytes : static_cast<cuuint64_t>(rows) * row_bytes};
    cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), static_cast<cuuint32_t>(box_planes)};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims, strides,
                          box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? TFA_OK : drv_fail("cuTensorMapEncodeTiled", static_cast<int>(r));
}

// How K/V (and Q/O) rows are addressed beyond the dense [B, H, len, D] layout.
struct Addressing {
    int ring_rows = 0;  // rotating cache: K/V [B, Hkv, ring_rows, D], key j in row j mod ring_rows
    const int *cu_q = nullptr, *cu_k = nullptr;  // packed variable-length batch (device, [B+1])
    int total_q = 0, total_k = 0;
    float *lse = nullptr;  // optional per-row log-sum-exp output (dense layout only)
};

template <int D>
int launch(DeviceState &st, const void *q, const void *k, const void *v, void *o, int B, int Hq,
           int Hkv, int L, int S, float scale, int causal, int window, const float *key_mask,
           cudaStream_t stream, unsigned flags, SplitScratch *ss, bool force_split = false,
           bool packed = false, float softcap = 0.f, const float *sinks = nullptr,
           const Addressing &ad = Addressing{}) {
    using C = tfa::Cfg<D>;
    // Short queries: a tile packs pack_heads query heads of one KV group, all L
    // rows of each (pack_heads * L <= 128), loaded as one {64, L, pack_heads} box.
    // Any call with L <= 128 has one query tile per item, so it runs packed:
    // the tile fills with more heads where L <= 64, and the packed schedule
    // double-buffers the score tile, which a single-tile item cannot use
    // otherwise.  (Variable-length batches keep per-sequence tiles.)
    const bool varlen = ad.cu_q != nullptr;
    if (!varlen && L <= tfa::kBlockQ) packed = true;
    const int G = Hq / Hkv;
    const int pack_heads = packed ? (G < tfa::kBlockQ / L ? G : tfa::kBlockQ / L) : 0;
    const int pack_chunks = packed ? (G + pack_heads - 1) / pack_heads : 0;
    CUtensorMap mq, mk, mv;
    int rc = 0;
    if (varlen)  // packed [total, H, D]: rows are tokens, planes are heads
        rc = encode_map(&mq, q, ad.total_q, Hq, D, tfa::kBlockQ, 1, true) ||
             encode_map(&mk, k, ad.total_k, Hkv, D, tfa::kBlockK, 1, true) ||
             encode_map(&mv, v, ad.total_k, Hkv, D, tfa::kBlockK, 1, true);
    else if (ad.ring_rows)  // K/V tiles arrive as two 64-row boxes (a box never wraps)
        rc = (packed ? encode_map(&mq, q, L, B * Hq, D, L, pack_heads) : encode_map(&mq, q, L, B * Hq, D)) ||
             encode_map(&mk, k, ad.ring_rows, B * Hkv, D, 64) || encode_map(&mv, v, ad.ring_rows, B * Hkv, D, 64);
    else
        rc = (packed ? encode_map(&mq, q, L, B * Hq, D, L, pack_heads) : encode_map(&mq, q, L, B * Hq, D)) ||
             encode_map(&mk, k, S, B * Hkv, D) || encode_map(&mv, v, S, B * Hkv, D);
    if (rc) return TFA_ERR_CUDA;
    // separate instantiations with and without a key mask (the mask costs an
    // extra MMA per score tile and extra shared memory), a softcap (extra work
    // per score) and the log-sum-exp output; plain calls carry none of them
    const bool sc = softcap > 0.f;
    if (sc && ad.lse) return TFA_ERR_SOFTCAP;  // no variant computes both (the backward has no softcap)
    const int mode = ad.lse ? tfa::kModeLse : sc ? tfa::kModeSoftcap : tfa::kModePlain;
    const int layout = varlen ? tfa::kLayoutVarlen : ad.ring_rows ? tfa::kLayoutRing : tfa::kLayoutDense;
    if (layout != tfa::kLayoutDense && (key_mask || ad.lse)) return TFA_ERR_RING;  // not instantiated
    if (varlen && packed) return TFA_ERR_RING;  // not instantiated
    using Kern = void (*)(const CUtensorMap, const CUtensorMap, const CUtensorMap, const tfa::Params);
    using namespace tfa;
#define TFA_DENSE(PK)                                                                               \
    {{tfa_prefill_kernel<D, false, kModePlain, kLayoutDense, PK>,                                   \
      tfa_prefill_kernel<D, true, kModePlain, kLayoutDense, PK>},                                   \
     {tfa_prefill_kernel<D, false, kModeSoftcap, kLayoutDense, PK>,                                 \
      tfa_prefill_kernel<D, true, kModeSoftcap, kLayoutDense, PK>},                                 \
     {tfa_prefill_kernel<D, false, kModeLse, kLayoutDense, PK>, tfa_prefill_kernel<D, true, kModeLse, kLayoutDense, PK>}}
    static const Kern dense[2][3][2] = {TFA_DENSE(false), TFA_DENSE(true)};  // [packed][mode][key mask]
#undef TFA_DENSE
    static const Kern ring[2][2] = {  // [packed][plain, softcap]
        {tfa_prefill_kernel<D, false, kModePlain, kLayoutRing, false>,
         tfa_prefill_kernel<D, false, kModeSoftcap, kLayoutRing, false>},
        {tfa_prefill_kernel<D, false, kModePlain, kLayoutRing, true>,
         tfa_prefill_kernel<D, false, kModeSoftcap, kLayoutRing, true>}};
    static const Kern vlen[2] = {tfa_prefill_kernel<D, false, kModePlain, kLayoutVarlen, false>,
                                 tfa_prefill_kernel<D, false, kModeSoftcap, kLayoutVarlen, false>};
    const Kern kern = layout == kLayoutDense ? dense[packed ? 1 : 0][mode][key_mask ? 1 : 0]
                      : layout == kLayoutRing ? ring[packed ? 1 : 0][sc ? 1 : 0]
                                              : vlen[sc ? 1 : 0];
    const int smem = key_mask ? C::kSmemBytesKeyMask : varlen ? C::kSmemBytesVarlen : C::kSmemBytes;
    const int which = variant_index(D, key_mask != nullptr, mode, layout, packed);
    if (!st.smem_attr[which]) return drv_fail("kernel not prepared", which);
    tfa::Params p;
    p.o = static_cast<__nv_bfloat16 *>(o);
    p.key_mask = key_mask;
    p.status = st.status;
    p.B = B;
    p.Hq = Hq;
    p.Hkv = Hkv;
    p.L = L;
    p.S = S;
    p.G = Hq / Hkv;
    p.causal = causal ? 1 : 0;
    p.window = (causal && window > 0) ? window : 0;
    p.flags = flags & (tfa::kFlagNoTileSkip | tfa::kFlagMaskAll);
    p.wait_limit = (flags & TFA_DEBUG_SHORT_WAITS) ? tfa::TFA_SHORT_WAIT_CYCLES : tfa::TFA_WAIT_LIMIT_CYCLES;
    p.scale_log2 = scale * 1.4426950408889634f;
    // softcap: y = b (1 - 2 / (2^(a x) + 1)) with a = 2 scale log2(e) / cap, b = cap / scale
    p.softcap_a = sc ? 2.f * scale * 1.4426950408889634f / softcap : 0.f;
    p.softcap_b = sc ? softcap / scale : 0.f;
    p.softcap_u = sc ? scale / softcap : 0.f;
    p.sinks = sinks;
    p.ring_rows = ad.ring_rows;
    p.total_q = ad.total_q;
    p.total_k = ad.total_k;
    p.cu_q = ad.cu_q;
    p.cu_k = ad.cu_k;
    p.lse = ad.lse;
    p.packed = packed ? 1 : 0;
    p.pack_heads = pack_heads;
    p.pack_chunks = pack_chunks;
    tfa::Shape &sh = p.shape;
    sh.B = B;
    sh.Hq = packed ? Hkv * pack_chunks : Hq;  // one "virtual head" per packed tile
    sh.L = L;
    sh.S = S;
    sh.causal = p.causal;
    sh.window = p.window;
    sh.flags = p.flags;
    sh.n_qp = tfa::shape_n_qp(L);
    p.W = varlen ? 0 : tfa::total_steps(sh);  // varlen: per-sequence lengths live on the device
    // Head pairs for causal calls whose items are short (at most 16 key tiles
    // on average) when a KV group has an even number of query heads: a pair of
    // consecutive query tiles spends one step on the later tile alone (the
    // diagonal, or the window's shift), which short items do not amortise;
    // measured, long items ran slower as head pairs.
    // (Variable-length batches: lengths unknown here, so when the longest
    // sequence has at most 32 query tiles.)
    if (!packed && p.causal && (Hq / Hkv) % 2 == 0 &&
        (varlen ? L <= 32 * tfa::kBlockQ : p.W <= 16LL * B * sh.Hq * sh.n_qp)) {
        sh.hp = 1;
        sh.Hq = Hq / 2;
        sh.n_qp = tfa::shape_n_qp(L, 1);
        if (!varlen) p.W = tfa::total_steps(sh);
    }
    const long long n_items = static_cast<long long>(B) * sh.Hq * sh.n_qp;
    // whole-item schedule, and the split one when scratch exists and the
    // estimate says it finishes sooner (few, large items per CTA)
    sh.split = 0;
    sh.grid = n_items < st.sm_count ? static_cast<int>(n_items) : st.sm_count;
    if (varlen) ss = nullptr;  // whole items only (the host does not know the lengths)
    if (ss != nullptr && (n_items <= (1 << 16) || force_split)) {
        tfa::Shape sp = sh;
        sp.split = 1;
        sp.grid = p.W < st.sm_count ? static_cast<int>(p.W) : st.sm_count;
        if (force_split || tfa::makespan_estimate(sp, p.W) < tfa::makespan_estimate(sh, p.W)) sh = sp;
    }
    if (!sh.split) ss = nullptr;
    p.partial = ss ? ss->partial : nullptr;
    p.ready = ss ? ss->ready : nullptr;
    p.ctl = ss ? ss->ctl : nullptr;
    if (sh.split) {
        // A split-schedule finalizer waits for flags that later CTAs of the grid
        // set, which needs every CTA resident at once (one per SM).  A cooperative
        // launch guarantees that or fails at once (an MPS SM limit, a green
        // context, another kernel holding SMs cannot make it wait forever); the
        // call then runs the whole-item schedule, which has no waits between CTAs.
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(static_cast<unsigned>(sh.grid));
        cfg.blockDim = dim3(tfa::kThreads);
        cfg.dynamicSmemBytes = static_cast<size_t>(smem);
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeCooperative;
        attr[0].val.cooperative = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, mq, mk, mv, p);
        if (e == cudaSuccess) return TFA_OK;
        if (e != cudaErrorCooperativeLaunchTooLarge) return cuda_fail("kernel launch (cooperative)", e);
        (void)cudaGetLastError();  // not sticky; clear it and deal whole items instead
        sh.split = 0;
        sh.grid = n_items < st.sm_count ? static_cast<int>(n_items) : st.sm_count;
        p.partial = nullptr;
        p.ready = nullptr;
        p.ctl = nullptr;
    }
    kern<<<sh.grid, tfa::kThreads, smem, stream>>>(mq, mk, mv, p);
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? TFA_OK : cuda_fail("kernel launch", e);
}

int prefill_impl(const void *q, const void *k, const void *v, void *o, int B, int Hq, int Hkv,
                 int L, int S, int D, float scale, int causal, int window, const float *key_mask,
                 cudaStream_t stream, unsigned flags) {
    int rc = validate(q, k, v, o, B, Hq, Hkv, L, S, D, scale, causal, window, key_mask, true);
    if (rc) return rc;
    if (flags & ~(TFA_DEBUG_NO_TILE_SKIP | TFA_DEBUG_MASK_ALL | TFA_DEBUG_SYNC | TFA_DEBUG_NO_SPLIT |
                  TFA_DEBUG_FORCE_SPLIT | TFA_DEBUG_SHORT_WAITS) ||
        ((flags & TFA_DEBUG_NO_SPLIT) && (flags & TFA_DEBUG_FORCE_SPLIT)))
        return TFA_ERR_FLAGS;
    const bool force_split = (flags & TFA_DEBUG_FORCE_SPLIT) != 0;
    DeviceState *st = nullptr;
    SplitScratch *ss = nullptr;
    std::lock_guard<std::mutex> lk(g_mutex);
    if ((rc = device_state(stream, &st))) return rc;
    if (!(flags & TFA_DEBUG_NO_SPLIT) && (rc = split_scratch(*st, stream, &ss))) return rc;
    const unsigned kflags = flags & (TFA_DEBUG_NO_TILE_SKIP | TFA_DEBUG_MASK_ALL | TFA_DEBUG_SHORT_WAITS);
    rc = (D == 128) ? launch<128>(*st, q, k, v, o, B, Hq, Hkv, L, S, scale, causal, window,
                                  key_mask, stream, kflags, ss, force_split)
                    : launch<64>(*st, q, k, v, o, B, Hq, Hkv, L, S, scale, causal, window,
                                 key_mask, stream, kflags, ss, force_split);
    if (rc) return rc;
    return TFA_OK;
}

int ensure_capacity(DeviceState &st, int i, size_t bytes) {
    if (st.h_cap[i] >= bytes) return TFA_OK;
    if (st.h_buf[i]) cudaFree(st.h_buf[i]);
    st.h_buf[i] = nullptr;
    st.h_cap[i] = 0;
    if (cudaMalloc(&st.h_buf[i], bytes) != cudaSuccess) return TFA_ERR_CUDA;
    st.h_cap[i] = bytes;
    return TFA_OK;
}

}  // namespace

extern "C" int tfa_prefill(const void *q, const void *k, const void *v, void *o, int B, int Hq,
                           int Hkv, int L, int S, int D, float scale, int causal, int window,
                           const float *key_mask, tfa_stream_t stream) {
    return prefill_impl(q, k, v, o, B, Hq, Hkv, L, S, D, scale, causal, window, key_mask,
                        reinterpret_cast<cudaStream_t>(stream), 0u);
}

extern "C" int tfa_decode(const void *q, const void *k, const void *v, void *o, int B, int Hq,
                          int Hkv, int L, int S, int D, float scale, int causal, int window,
                          const float *key_mask, tfa_stream_t stream) {
    int rc = validate(q, k, v, o, B, Hq, Hkv, L, S, D, scale, causal, window, key_mask, true, true);
    if (rc) return rc;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    DeviceState *st = nullptr;
    SplitScratch *ss = nullptr;
    std::lock_guard<std::mutex> lk(g_mutex);
    if ((rc = device_state(s, &st)) || (rc = split_scratch(*st, s, &ss))) return rc;
    return (D == 128) ? launch<128>(*st, q, k, v, o, B, Hq, Hkv, L, S, scale, causal, window,
                                    key_mask, s, 0u, ss, false, true)
                      : launch<64>(*st, q, k, v, o, B, Hq, Hkv, L, S, scale, causal, window,
                                   key_mask, s, 0u, ss, false, true);
}

extern "C" int tfa_attention_ex(const void *q, const void *k, const void *v, void *o, int B,
                                int Hq, int Hkv, int L, int S, int D, float scale, int causal,
                                int window, const float *key_mask, float softcap,
                                const float *sinks, tfa_stream_t stream) {
    const bool decode = L >= 1 && L <= TFA_MAX_DECODE_ROWS;
    int rc = validate(q, k, v, o, B, Hq, Hkv, L, S, D, scale, causal, window, key_mask, true, decode);
    if (rc) return rc;
    if (!std::isfinite(softcap) || softcap < 0.f || (softcap > 0.f && scale == 0.f)) return TFA_ERR_SOFTCAP;
    if (sinks && (reinterpret_cast<uintptr_t>(sinks) & 3u)) return TFA_ERR_ALIGN;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    DeviceState *st = nullptr;
    SplitScratch *ss = nullptr;
    std::lock_guard<std::mutex> lk(g_mutex);
    if ((rc = device_state(s, &st)) || (rc = split_scratch(*st, s, &ss))) return rc;
    return (D == 128) ? launch<128>(*st, q, k, v, o, B, Hq, Hkv, L, S, scale, causal, window,
                                    key_mask, s, 0u, ss, false, decode, softcap, sinks)
                      : launch<64>(*st, q, k, v, o, B, Hq, Hkv, L, S, scale, causal, window,
                                   key_mask, s, 0u, ss, false, decode, softcap, sinks);
}

extern "C" int tfa_prefill_ring(const void *q, const void *k, const void *v, void *o, int B,
                                int Hq, int Hkv, int L, int S, int ring_rows, int D, float scale,
                                int window, float softcap, const float *sinks, tfa_stream_t stream) {
    const bool decode = L >= 1 && L <= TFA_MAX_DECODE_ROWS;
    int rc = validate(q, k, v, o, B, Hq, Hkv, L, S, D, scale, 1, window, nullptr, true, decode);
    if (rc) return rc;
    if (window <= 0 || ring_rows < 64 || ring_rows % 64 != 0 ||
        static_cast<long long>(ring_rows) < static_cast<long long>(window) - 1 + L ||
        static_cast<long long>(B) * Hkv * ring_rows > (1ll << 31) - 1)
        return TFA_ERR_RING;
    if (!std::isfinite(softcap) || softcap < 0.f || (softcap > 0.f && scale == 0.f)) return TFA_ERR_SOFTCAP;
    if (sinks && (reinterpret_cast<uintptr_t>(sinks) & 3u)) return TFA_ERR_ALIGN;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    DeviceState *st = nullptr;
    SplitScratch *ss = nullptr;
    std::lock_guard<std::mutex> lk(g_mutex);
    if ((rc = device_state(s, &st)) || (rc = split_scratch(*st, s, &ss))) return rc;
    Addressing ad;
    ad.ring_rows = ring_rows;
    return (D == 128) ? launch<128>(*st, q, k, v, o, B, Hq, Hkv, L, S, scale, 1, window, nullptr, s, 0u,
                                    ss, false, decode, softcap, sinks, ad)
                      : launch<64>(*st, q, k, v, o, B, Hq, Hkv, L, S, scale, 1, window, nullptr, s, 0u,
                                   ss, false, decode, softcap, sinks, ad);
}

extern "C" int tfa_prefill_varlen(const void *q, const void *k, const void *v, void *o,
                                  const int *cu_seqlens_q, const int *cu_seqlens_k, int B, int Hq,
                                  int Hkv, int total_q, int total_k, int max_seqlen_q, int D,
                                  float scale, int causal, int window, float softcap,
                                  const float *sinks, tfa_stream_t stream) {
    if (total_q == 0) return TFA_OK;  // no query row: nothing is read or written
    if (!q || !k || !v || !o || !cu_seqlens_q || !cu_seqlens_k) return TFA_ERR_NULL;
    if (Hq < 1 || Hkv < 1 || Hq % Hkv != 0) return TFA_ERR_HEADS;
    if (B < 1 || B > tfa::kMaxVarlenSeqs || total_q < 0 || total_k < 0 || max_seqlen_q < 0 ||
        max_seqlen_q > (1 << 30) || static_cast<long long>(total_q) * Hq > (1ll << 31) - 1 ||
        static_cast<long long>(total_k) * Hkv > (1ll << 31) - 1)
        return TFA_ERR_SHAPE;
    if (D != 64 && D != 128) return TFA_ERR_HEAD_DIM;
    if (window > 0 && !causal) return TFA_ERR_WINDOW;
    auto mis = [](const void *p, unsigned a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) != 0; };
    if (mis(q, 16) || mis(k, 16) || mis(v, 16) || mis(o, 16) || mis(cu_seqlens_q, 4) ||
        mis(cu_seqlens_k, 4) || (sinks && mis(sinks, 4)))
        return TFA_ERR_ALIGN;
    if (!std::isfinite(scale)) return TFA_ERR_SCALE;
    if (!std::isfinite(softcap) || softcap < 0.f || (softcap > 0.f && scale == 0.f)) return TFA_ERR_SOFTCAP;
    if (max_seqlen_q == 0) return TFA_ERR_SHAPE;  // query rows exist, so some sequence has one
    if (total_k == 0) return TFA_ERR_SHAPE;  // keys are read through a map over k: it needs rows
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    DeviceState *st = nullptr;
    std::lock_guard<std::mutex> lk(g_mutex);
    int rc = device_state(s, &st);
    if (rc) return rc;
    Addressing ad;
    ad.cu_q = cu_seqlens_q;
    ad.cu_k = cu_seqlens_k;
    ad.total_q = total_q;
    ad.total_k = total_k;
    return (D == 128) ? launch<128>(*st, q, k, v, o, B, Hq, Hkv, max_seqlen_q, max_seqlen_q, scale,
                                    causal, window, nullptr, s, 0u, nullptr, false, false, softcap,
                                    sinks, ad)
                      : launch<64>(*st, q, k, v, o, B, Hq, Hkv, max_seqlen_q, max_seqlen_q, scale,
                                   causal, window, nullptr, s, 0u, nullptr, false, false, softcap,
                                   sinks, ad);
}

namespace {
// Backward: a forward recompute (output and log-sum-exp into the workspace),
// delta = rowsum(dO o O), then the dQ and the dK/dV kernels, all on `stream`.
// o_saved / lse_saved: the forward's output and per-row log-sum-exp (as
// tfa_prefill_lse writes them), or nullptr to recompute both into the workspace.
template <int D>
int backward_impl(DeviceState &st, SplitScratch *ss, BwdScratch &bs, const void *q, const void *k,
                  const void *v, const void *dout, void *dq, void *dk, void *dv, int B, int Hq,
                  int Hkv, int L, int S, float scale, int causal, int window, const float *key_mask,
                  cudaStream_t stream, const void *o_saved = nullptr, const float *lse_saved = nullptr) {
    namespace bw = tfa::bwd;
    const void *o = o_saved;
    const float *lse = lse_saved;
    if (!o) {
        const bool decode = L <= TFA_MAX_DECODE_ROWS;
        Addressing ad;
        ad.lse = bs.lse;
        const int rc = launch<D>(st, q, k, v, bs.o, B, Hq, Hkv, L, S, scale, causal, window, key_mask, stream,
                                 0u, ss, false, decode, 0.f, nullptr, ad);
        if (rc) return rc;
        o = bs.o;
        lse = bs.lse;
    }
    const long long rows = static_cast<long long>(B) * Hq * L;
    const long long threads = rows * 32;
    bw::delta_kernel<D><<<static_cast<unsigned>((threads + 255) / 256), 256, 0, stream>>>(
        static_cast<const __nv_bfloat16 *>(o), static_cast<const __nv_bfloat16 *>(dout), bs.delta, rows);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail("delta kernel launch", e);
    CUtensorMap mq, mdo, mk, mv;
    if (encode_map(&mq, q, L, B * Hq, D) || encode_map(&mdo, dout, L, B * Hq, D) ||
        encode_map(&mk, k, S, B * Hkv, D) || encode_map(&mv, v, S, B * Hkv, D))
        return TFA_ERR_CUDA;
    if (!st.bwd_attr[(D == 128 ? 2 : 0) + (key_mask ? 1 : 0)]) return drv_fail("backward kernel not prepared", D);
    bw::BwdParams p;
    p.dq = static_cast<__nv_bfloat16 *>(dq);
    p.dk = static_cast<__nv_bfloat16 *>(dk);
    p.dv = static_cast<__nv_bfloat16 *>(dv);
    p.lse = lse;
    p.delta = bs.delta;
    p.key_mask = key_mask;
    p.status = st.status;
    p.B = B;
    p.Hq = Hq;
    p.Hkv = Hkv;
    p.L = L;
    p.S = S;
    p.G = Hq / Hkv;
    p.causal = causal ? 1 : 0;
    p.window = (causal && window > 0) ? window : 0;
    p.scale = scale;
    p.scale_log2 = scale * 1.4426950408889634f;
    const int smem = bw::Cfg<D>::kSmemBytes;
    const long long nq_items = static_cast<long long>(B) * Hq * ((L + tfa::kBlockQ - 1) / tfa::kBlockQ);
    p.n_items = static_cast<int>(nq_items);
    auto dq_kern = key_mask ? bw::dq_kernel<D, true> : bw::dq_kernel<D, false>;
    dq_kern<<<static_cast<int>(nq_items < st.sm_count ? nq_items : st.sm_count), bw::kThreads, smem, stream>>>(
        mq, mdo, mk, mv, p);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail("dQ kernel launch", e);
    const long long nk_items = static_cast<long long>(B) * Hkv * ((S + tfa::kBlockK - 1) / tfa::kBlockK);
    p.n_items = static_cast<int>(nk_items);
    auto dkv_kern = key_mask ? bw::dkv_kernel<D, true> : bw::dkv_kernel<D, false>;
    // Programmatic stream serialisation: the dK/dV CTAs start on the SMs the
    // dQ kernel's CTAs leave (the two kernels are independent; dK/dV waits for
    // dQ's completion only before it exits).
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(nk_items < st.sm_count ? nk_items : st.sm_count));
    cfg.blockDim = dim3(bw::kThreads);
    cfg.dynamicSmemBytes = static_cast<size_t>(smem);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if ((e = cudaLaunchKernelEx(&cfg, dkv_kern, mq, mdo, mk, mv, p)) != cudaSuccess)
        return cuda_fail("dK/dV kernel launch", e);
    return TFA_OK;
}
}  // namespace

extern "C" int tfa_prefill_backward(const void *q, const void *k, const void *v, const void *dout,
                                    void *dq, void *dk, void *dv, int B, int Hq, int Hkv, int L,
                                    int S, int D, float scale, int causal, int window,
                                    const float *key_mask, tfa_stream_t stream) {
    const bool decode = L >= 1 && L <= TFA_MAX_DECODE_ROWS;
    int rc = validate(q, k, v, dout, B, Hq, Hkv, L, S, D, scale, causal, window, key_mask, true, decode);
    if (rc) return rc;
    if (!dq || !dk || !dv) return TFA_ERR_NULL;
    auto mis16 = [](const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) != 0; };
    if (mis16(dq) || mis16(dk) || mis16(dv)) return TFA_ERR_ALIGN;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    DeviceState *st = nullptr;
    SplitScratch *ss = nullptr;
    BwdScratch *bs = nullptr;
    std::lock_guard<std::mutex> lk(g_mutex);
    if ((rc = device_state(s, &st)) || (rc = split_scratch(*st, s, &ss)) ||
        (rc = bwd_scratch(*st, s, static_cast<size_t>(B) * Hq * L, D, &bs)))
        return rc;
    return (D == 128) ? backward_impl<128>(*st, ss, *bs, q, k, v, dout, dq, dk, dv, B, Hq, Hkv, L, S, scale,
                                           causal, window, key_mask, s)
                      : backward_impl<64>(*st, ss, *bs, q, k, v, dout, dq, dk, dv, B, Hq, Hkv, L, S, scale,
                                          causal, window, key_mask, s);
}

extern "C" int tfa_prefill_lse(const void *q, const void *k, const void *v, void *o, float *lse, int B,
                               int Hq, int Hkv, int L, int S, int D, float scale, int causal, int window,
                               const float *key_mask, tfa_stream_t stream) {
    const bool decode = L >= 1 && L <= TFA_MAX_DECODE_ROWS;
    int rc = validate(q, k, v, o, B, Hq, Hkv, L, S, D, scale, causal, window, key_mask, true, decode);
    if (rc) return rc;
    if (!lse) return TFA_ERR_NULL;
    if (reinterpret_cast<uintptr_t>(lse) & 3u) return TFA_ERR_ALIGN;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    DeviceState *st = nullptr;
    SplitScratch *ss = nullptr;
    std::lock_guard<std::mutex> lk(g_mutex);
    if ((rc = device_state(s, &st)) || (rc = split_scratch(*st, s, &ss))) return rc;
    Addressing ad;
    ad.lse = lse;
    return (D == 128) ? launch<128>(*st, q, k, v, o, B, Hq, Hkv, L, S, scale, causal, window, key_mask, s, 0u,
                                    ss, false, decode, 0.f, nullptr, ad)
                      : launch<64>(*st, q, k, v, o, B, Hq, Hkv, L, S, scale, causal, window, key_mask, s, 0u,
                                   ss, false, decode, 0.f, nullptr, ad);
}

extern "C" int tfa_prefill_backward_saved(const void *q, const void *k, const void *v, const void *o,
                                          const float *lse, const void *dout, void *dq, void *dk, void *dv,
                                          int B, int Hq, int Hkv, int L, int S, int D, float scale,
                                          int causal, int window, const float *key_mask, tfa_stream_t stream) {
    const bool decode = L >= 1 && L <= TFA_MAX_DECODE_ROWS;
    int rc = validate(q, k, v, dout, B, Hq, Hkv, L, S, D, scale, causal, window, key_mask, true, decode);
    if (rc) return rc;
    if (!o || !lse || !dq || !dk || !dv) return TFA_ERR_NULL;
    auto mis16 = [](const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) != 0; };
    if (mis16(o) || mis16(dq) || mis16(dk) || mis16(dv) || (reinterpret_cast<uintptr_t>(lse) & 3u))
        return TFA_ERR_ALIGN;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    DeviceState *st = nullptr;
    BwdScratch *bs = nullptr;
    std::lock_guard<std::mutex> lk(g_mutex);
    if ((rc = device_state(s, &st)) || (rc = bwd_scratch(*st, s, static_cast<size_t>(B) * Hq * L, D, &bs)))
        return rc;
    return (D == 128) ? backward_impl<128>(*st, nullptr, *bs, q, k, v, dout, dq, dk, dv, B, Hq, Hkv, L, S, scale,
                                           causal, window, key_mask, s, o, lse)
                      : backward_impl<64>(*st, nullptr, *bs, q, k, v, dout, dq, dk, dv, B, Hq, Hkv, L, S, scale,
                                          causal, window, key_mask, s, o, lse);
}

extern "C" int tfa_prefill_debug(const void *q, const void *k, const void *v, void *o, int B,
                                 int Hq, int Hkv, int L, int S, int D, float scale, int causal,
                                 int window, const float *key_mask, tfa_stream_t stream,
                                 unsigned flags) {
    const int rc = prefill_impl(q, k, v, o, B, Hq, Hkv, L, S, D, scale, causal, window, key_mask,
                                reinterpret_cast<cudaStream_t>(stream), flags);
    if (rc == TFA_OK && (flags & TFA_DEBUG_SYNC)) return tfa_check_status(stream);
    return rc;
}

extern "C" int tfa_prefill_host(const void *q, const void *k, const void *v, void *o, int B,
                                int Hq, int Hkv, int L, int S, int D, float scale, int causal,
                                int window, const float *key_mask, tfa_stream_t stream) {
    const bool decode = L >= 1 && L <= TFA_MAX_DECODE_ROWS;
    int rc = validate(q, k, v, o, B, Hq, Hkv, L, S, D, scale, causal, window, key_mask, true, decode);
    if (rc) return rc;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const size_t qbytes = static_cast<size_t>(B) * Hq * L * D * 2;
    const size_t kbytes = static_cast<size_t>(B) * Hkv * S * D * 2;
    const size_t mbytes = key_mask ? static_cast<size_t>(B) * S * sizeof(float) : 0;
    DeviceState *st = nullptr;
    std::lock_guard<std::mutex> lk(g_mutex);
    if ((rc = device_state(s, &st))) return rc;
    if ((rc = ensure_capacity(*st, 0, qbytes)) || (rc = ensure_capacity(*st, 1, kbytes)) ||
        (rc = ensure_capacity(*st, 2, kbytes)) || (rc = ensure_capacity(*st, 3, qbytes)) ||
        (mbytes && (rc = ensure_capacity(*st, 4, mbytes))))
        return rc;
    if (!st->h_in) {
        cudaError_t e = cudaStreamCreateWithFlags(&st->h_in, cudaStreamNonBlocking);
        if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&st->h_out, cudaStreamNonBlocking);
        for (int i = 0; i < 2 * kHostStages + 1 && e == cudaSuccess; ++i)
            e = cudaEventCreateWithFlags(&st->h_ev[i], cudaEventDisableTiming);
        if (e != cudaSuccess) return cuda_fail("tfa_prefill_host stream/event setup", e);
    }
    SplitScratch *ss = nullptr;
    if ((rc = split_scratch(*st, s, &ss))) return rc;
    // Pipeline stages over KV groups, which are contiguous in the
    // [B, H, rows, D] layouts (group g of batch b: query planes b Hq + g G ..,
    // KV plane b Hkv + g): stage i's inputs are copied in on h_in while stage
    // i - 1 computes on `stream` and stage i - 2's output is copied out on
    // h_out.  Up to kHostStages batch elements: ranges of groups inside one element;
    // beyond: runs of whole elements.
    const int G = Hq / Hkv;
    int per_b = 1, gps = Hkv, bps = 1;  // stages per element, groups per stage, elements per stage
    if (B <= kHostStages) {
        per_b = kHostStages / B < Hkv ? kHostStages / B : Hkv;
        gps = (Hkv + per_b - 1) / per_b;
        per_b = (Hkv + gps - 1) / gps;
    } else {
        bps = (B + kHostStages - 1) / kHostStages;
    }
    const int n_stages = B <= kHostStages ? B * per_b : (B + bps - 1) / bps;
    const size_t q_plane = static_cast<size_t>(L) * D * 2, k_plane = static_cast<size_t>(S) * D * 2;
    const char *hq = static_cast<const char *>(q), *hk = static_cast<const char *>(k),
               *hv = static_cast<const char *>(v);
    char *dq = static_cast<char *>(st->h_buf[0]), *dk = static_cast<char *>(st->h_buf[1]),
         *dv = static_cast<char *>(st->h_buf[2]), *dout = static_cast<char *>(st->h_buf[3]);
    const float *dmask = mbytes ? static_cast<const float *>(st->h_buf[4]) : nullptr;
    // the caller's earlier work on `stream` comes first
    if (cudaEventRecord(st->h_ev[2 * kHostStages], s) != cudaSuccess ||
        cudaStreamWaitEvent(st->h_in, st->h_ev[2 * kHostStages], 0) != cudaSuccess)
        return TFA_ERR_CUDA;
    if (mbytes && cudaMemcpyAsync(st->h_buf[4], key_mask, mbytes, cudaMemcpyHostToDevice, st->h_in) != cudaSuccess)
        return TFA_ERR_CUDA;
    for (int i = 0; i < n_stages; ++i) {
        // query planes [qp0, qp0 + nq), KV planes [kp0, kp0 + nk) of this stage; the
        // kernel sees them as Bs elements of Hs query and Hks KV heads
        int b0, Bs, Hs, Hks;
        size_t qp0, kp0;
        if (B <= kHostStages) {
            b0 = i / per_b;
            const int g0 = (i % per_b) * gps;
            const int ng = Hkv - g0 < gps ? Hkv - g0 : gps;
            Bs = 1;
            Hs = ng * G;
            Hks = ng;
            qp0 = static_cast<size_t>(b0) * Hq + static_cast<size_t>(g0) * G;
            kp0 = static_cast<size_t>(b0) * Hkv + g0;
        } else {
            b0 = i * bps;
            Bs = B - b0 < bps ? B - b0 : bps;
            Hs = Hq;
            Hks = Hkv;
            qp0 = static_cast<size_t>(b0) * Hq;
            kp0 = static_cast<size_t>(b0) * Hkv;
        }
        const size_t nq = static_cast<size_t>(Bs) * Hs, nk = static_cast<size_t>(Bs) * Hks;
        if (cudaMemcpyAsync(dq + qp0 * q_plane, hq + qp0 * q_plane, nq * q_plane, cudaMemcpyHostToDevice, st->h_in) !=
                cudaSuccess ||
            cudaMemcpyAsync(dk + kp0 * k_plane, hk + kp0 * k_plane, nk * k_plane, cudaMemcpyHostToDevice, st->h_in) !=
                cudaSuccess ||
            cudaMemcpyAsync(dv + kp0 * k_plane, hv + kp0 * k_plane, nk * k_plane, cudaMemcpyHostToDevice, st->h_in) !=
                cudaSuccess ||
            cudaEventRecord(st->h_ev[2 * i], st->h_in) != cudaSuccess ||
            cudaStreamWaitEvent(s, st->h_ev[2 * i], 0) != cudaSuccess)
            return TFA_ERR_CUDA;
        const float *smask = dmask ? dmask + static_cast<size_t>(b0) * S : nullptr;
        rc = (D == 128) ? launch<128>(*st, dq + qp0 * q_plane, dk + kp0 * k_plane, dv + kp0 * k_plane,
                                      dout + qp0 * q_plane, Bs, Hs, Hks, L, S, scale, causal, window, smask, s, 0u,
                                      ss, false, decode)
                        : launch<64>(*st, dq + qp0 * q_plane, dk + kp0 * k_plane, dv + kp0 * k_plane,
                                     dout + qp0 * q_plane, Bs, Hs, Hks, L, S, scale, causal, window, smask, s, 0u,
                                     ss, false, decode);
        if (rc) return rc;
        if (cudaEventRecord(st->h_ev[2 * i + 1], s) != cudaSuccess ||
            cudaStreamWaitEvent(st->h_out, st->h_ev[2 * i + 1], 0) != cudaSuccess ||
            cudaMemcpyAsync(static_cast<char *>(o) + qp0 * q_plane, dout + qp0 * q_plane, nq * q_plane,
                            cudaMemcpyDeviceToHost, st->h_out) != cudaSuccess)
            return TFA_ERR_CUDA;
    }
    if (cudaStreamSynchronize(st->h_out) != cudaSuccess || cudaStreamSynchronize(s) != cudaSuccess)
        return TFA_ERR_CUDA;
    return TFA_OK;
}

// ------------------------------------------------------------------------
// No-allocation variant.
//
// Some callers cannot call cudaMalloc at all: code that runs under a caching
// or arena allocator that owns all device memory, code that must not allocate
// while a graph is being recorded or while latency-critical work is running,
// and embedded runtimes that hand the library only their own buffers.  For
// them, tfa_prefill_noalloc runs the same kernel as tfa_prefill, but the
// kernel's scratch (its status word) lives in this file-scope device array,
// which every GPU that loads the library holds until the process exits.  In
// host code the array's name is only a host-side stand-in, never a device
// address: its real address is looked up with cudaGetSymbolAddress once per
// device, with that device current, and passed to the kernel.
constexpr size_t kNoAllocScratchBytes = 256;            // the stated maximum
constexpr size_t kKernelScratchBytes = sizeof(unsigned);  // what the kernel needs, for every size
static_assert(kKernelScratchBytes <= kNoAllocScratchBytes, "the kernel's scratch must fit the static array");
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {
DeviceState g_noalloc_dev[kMaxDevices];  // set up by the first tfa_prefill_noalloc per device

int noalloc_state(cudaStream_t stream, DeviceState **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail("cudaGetDevice", e);
    if (dev < 0 || dev >= kMaxDevices) return drv_fail("device index out of range", dev);
    DeviceState &st = g_noalloc_dev[dev];
    if (!st.init) {
        // the set-up below clears the array with a memset that a capture would
        // record instead of running
        if (int rc = refuse_under_capture(stream, "the no-alloc scratch")) return rc;
        void *ptr = nullptr;
        if ((e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch)) != cudaSuccess)
            return cuda_fail("cudaGetSymbolAddress(no-alloc scratch)", e);
        // the status word must start at zero; clearing is not an allocation
        if ((e = cudaMemsetAsync(ptr, 0, kNoAllocScratchBytes, stream)) != cudaSuccess)
            return cuda_fail("cudaMemsetAsync(no-alloc scratch)", e);
        if ((e = cudaDeviceGetAttribute(&st.sm_count, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
            return cuda_fail("cudaDeviceGetAttribute", e);
        if (int rc = get_encode_fn()) return rc;
        if (int rc = prepare_all_kernels(st)) return rc;
        st.status = static_cast<unsigned *>(ptr);
        st.init = true;
    }
    *out = &st;
    return TFA_OK;
}

// Reads and clears one status word (synchronous); TFA_OK, TFA_ERR_TIMEOUT or TFA_ERR_CUDA.
int take_status_word(unsigned *status) {
    unsigned word = 0;
    if (cudaMemcpy(&word, status, sizeof word, cudaMemcpyDeviceToHost) != cudaSuccess)
        return TFA_ERR_CUDA;
    if (word == 0) return TFA_OK;
    if (cudaMemset(status, 0, sizeof word) != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess)
        return TFA_ERR_CUDA;
    return (word & tfa::TFA_DEVICE_TIMEOUT) ? TFA_ERR_TIMEOUT : TFA_ERR_SEQLENS;
}
}  // namespace

extern "C" int tfa_prefill_noalloc(const void *q, const void *k, const void *v, void *o, int B,
                                   int Hq, int Hkv, int L, int S, int D, float scale, int causal,
                                   int window, const float *key_mask, tfa_stream_t stream) {
    int rc = validate(q, k, v, o, B, Hq, Hkv, L, S, D, scale, causal, window, key_mask, true);
    if (rc) return rc;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    DeviceState *st = nullptr;
    std::lock_guard<std::mutex> lk(g_mutex);
    if ((rc = noalloc_state(s, &st))) return rc;
    // whole-item schedule: the split schedule's partials would not fit the static array
    return (D == 128) ? launch<128>(*st, q, k, v, o, B, Hq, Hkv, L, S, scale, causal, window,
                                    key_mask, s, 0u, nullptr)
                      : launch<64>(*st, q, k, v, o, B, Hq, Hkv, L, S, scale, causal, window,
                                   key_mask, s, 0u, nullptr);
}

extern "C" int tfa_check_status(tfa_stream_t stream) {
    if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return TFA_ERR_CUDA;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return TFA_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_mutex);
    // read and clear both words every time, so that neither is left set and
    // blamed on later calls; a timeout in either one wins
    const int a = g_dev[dev].init ? take_status_word(g_dev[dev].status) : TFA_OK;
    const int b = g_noalloc_dev[dev].init ? take_status_word(g_noalloc_dev[dev].status) : TFA_OK;
    if (a == TFA_ERR_CUDA || b == TFA_ERR_CUDA) return TFA_ERR_CUDA;
    if (a == TFA_ERR_TIMEOUT || b == TFA_ERR_TIMEOUT) return TFA_ERR_TIMEOUT;
    return a != TFA_OK ? a : b;
}

extern "C" const char *tfa_last_error(void) { return g_last_error; }

#ifdef TFA_TRACE
// Trace builds only: copy CTA 0's timeline (4 roles x kTraceSlots clocks) to host.
extern "C" int tfa_trace_read(unsigned long long *host, size_t n) {
    const size_t bytes = sizeof(tfa::g_tfa_trace);
    if (n * sizeof(unsigned long long) < bytes) return TFA_ERR_SHAPE;
    cudaError_t e = cudaMemcpyFromSymbol(host, tfa::g_tfa_trace, bytes);
    return e == cudaSuccess ? TFA_OK : cuda_fail("cudaMemcpyFromSymbol(trace)", e);
}
// Trace builds only: per-CTA global-timer stamps (1024 x 4: start, end, pieces done, spare).
extern "C" int tfa_trace_cta_times(unsigned long long *host, size_t n) {
    const size_t bytes = sizeof(tfa::g_tfa_cta_time);
    if (n * sizeof(unsigned long long) < bytes) return TFA_ERR_SHAPE;
    cudaError_t e = cudaMemcpyFromSymbol(host, tfa::g_tfa_cta_time, bytes);
    return e == cudaSuccess ? TFA_OK : cuda_fail("cudaMemcpyFromSymbol(cta times)", e);
}
#endif

extern "C" const char *tfa_status_string(int status) {
    switch (status) {
        case TFA_OK: return "ok";
        case TFA_ERR_NULL: return "a tensor pointer is NULL";
        case TFA_ERR_HEADS: return "query heads must be a positive multiple of KV heads";
        case TFA_ERR_SHORT_QUERY: return "query shorter than the tiled operator's minimum (9 rows)";
        case TFA_ERR_SHAPE: return "invalid shape (B < 1, S < L, or sizes out of range)";
        case TFA_ERR_HEAD_DIM: return "head dimension must be 64 or 128";
        case TFA_ERR_WINDOW: return "a sliding window requires causal attention";
        case TFA_ERR_ALIGN: return "tensor pointers must be 16-byte aligned (key mask 4-byte)";
        case TFA_ERR_CUDA: return "a CUDA call failed";
        case TFA_ERR_TIMEOUT: return "a kernel wait timed out; the output is invalid";
        case TFA_ERR_SCALE: return "scale must be finite";
        case TFA_ERR_CAPTURE: return "first use of a device or stream inside a CUDA graph capture";
        case TFA_ERR_SOFTCAP: return "softcap must be finite and >= 0 (and needs a nonzero scale)";
        case TFA_ERR_SEQLENS: return "inconsistent cu_seqlens in a variable-length call; its output is invalid";
        case TFA_ERR_RING: return "ring cache needs a window, ring_rows a multiple of 64 and >= window - 1 + L";
        case TFA_ERR_FLAGS: return "unknown debug flags";
        default: return "unknown status";
    }
}

extern "C" int tfa_plan_ktile(int L, int S, int causal, int window, int ktile, int *qt_lo,
                              int *qt_hi) {
    int rc = validate(nullptr, nullptr, nullptr, nullptr, 1, 1, 1, L, S, 128, 1.0f, causal, window,
                      nullptr, false, L < TFA_MIN_QUERY_ROWS);
    if (rc) return rc;
    if (!qt_lo || !qt_hi) return TFA_ERR_NULL;
    if (ktile < 0 || ktile * tfa::kBlockK >= S) return TFA_ERR_SHAPE;
    const tfa::KeyRange r = tfa::ktile_query_range(L, S, causal, causal ? window : 0, ktile);
    *qt_lo = r.lo;
    *qt_hi = r.hi;
    return TFA_OK;
}

extern "C" int tfa_plan_qtile(int L, int S, int causal, int window, int has_key_mask, int qtile,
                              int *kt_lo, int *kt_hi, unsigned char *needs_mask, int needs_mask_len) {
    int rc = validate(nullptr, nullptr, nullptr, nullptr, 1, 1, 1, L, S, 128, 1.0f, causal, window,
                      nullptr, false, L < TFA_MIN_QUERY_ROWS);
    if (rc) return rc;
    if (!kt_lo || !kt_hi) return TFA_ERR_NULL;
    const int q0 = qtile * tfa::kBlockQ;
    if (qtile < 0 || q0 >= L) return TFA_ERR_SHAPE;
    const tfa::KeyRange r = tfa::qtile_key_range(L, S, causal, causal ? window : 0, q0, 0u);
    *kt_lo = r.lo;
    *kt_hi = r.hi;
    if (needs_mask) {
        if (needs_mask_len < r.hi - r.lo + 1) return TFA_ERR_SHAPE;
        for (int j = r.lo; j <= r.hi; ++j)
            needs_mask[j - r.lo] = tfa::key_tile_needs_mask(L, S, causal, causal ? window : 0,
                                                            has_key_mask, q0, j, 0u) ? 1 : 0;
    }
    return TFA_OK;
}

extern "C" int tfa_plan_pieces(int B, int Hq, int L, int S, int causal, int window, int grid,
                               int split, int cta, int *out, int max_pieces, int *n_pieces,
                               long long *total_steps) {
    int rc = validate(nullptr, nullptr, nullptr, nullptr, B, Hq, Hq, L, S, 128, 1.0f, causal,
                      window, nullptr, false);
    if (rc) return rc;
    if (!n_pieces || (max_pieces > 0 && !out)) return TFA_ERR_NULL;
    tfa::Shape sh;
    sh.hp = (split & 2) ? 1 : 0;
    if (sh.hp && Hq % 2) return TFA_ERR_SHAPE;
    sh.B = B;
    sh.Hq = sh.hp ? Hq / 2 : Hq;
    sh.L = L;
    sh.S = S;
    sh.causal = causal ? 1 : 0;
    sh.window = (causal && window > 0) ? window : 0;
    sh.flags = 0;
    sh.n_qp = tfa::shape_n_qp(L, sh.hp);
    sh.split = (split & 1) ? 1 : 0;
    sh.grid = grid;
    const long long W = tfa::total_steps(sh);
    if (total_steps) *total_steps = W;
    const long long units = sh.split ? W : static_cast<long long>(B) * sh.Hq * sh.n_qp;
    if (grid < 1 || grid > units || cta < 0 || cta >= grid) return TFA_ERR_SHAPE;
    tfa::SegIter it;
    it.init(sh, W, cta);
    tfa::Segment seg;
    int n = 0;
    while (it.next(sh, seg)) {
        if (n < max_pieces) {
            const tfa::ItemSpan sp = tfa::item_span(sh, seg.qp);
            int *o = out + 10 * n;
            o[0] = seg.item;
            o[1] = seg.qp;
            o[2] = seg.b;
            o[3] = seg.h;
            o[4] = seg.jb;
            o[5] = seg.je;
            for (int t = 0; t < 2; ++t) {
                const tfa::TileRole tr = tfa::tile_role(sh, seg, sp, t);
                o[6 + t] = (tr.active ? 1 : 0) | (tr.finalizer ? 2 : 0) | (tr.complete ? 4 : 0);
                o[8 + t] = (tr.active && tr.finalizer && !tr.complete)
                               ? tfa::last_contributor(W, grid, cta, seg, sp, t)
                               : -1;
            }
        }
        ++n;
    }
    *n_pieces = n;
    return n <= max_pieces ? TFA_OK : TFA_ERR_SHAPE;
}
