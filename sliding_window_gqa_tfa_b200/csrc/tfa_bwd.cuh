// tfa_bwd.cuh -- backward pass of tiled GQA prefill attention on sm_100a:
// dQ, dK and dV of the bare attention core, recompute-based (brotensor
// "include/brotensor/ops/flash_attention.h", flash_attention_backward: no
// forward caches are consumed; causal- and mask-excluded positions contribute
// nothing to any gradient).  With s = q.k (raw), c = scale * log2(e),
// lse the per-row base-2 log-sum-exp of s*c (from a forward recompute) and
// delta_i = sum_d dO[i,d] O[i,d]:
//   P[i,j]  = 2^(s[i,j] c - lse_i)                (0 where (i, j) is excluded)
//   dP[i,j] = dO[i] . V[j]
//   dS[i,j] = P[i,j] (dP[i,j] - delta_i)
//   dQ[i]   = scale sum_j dS[i,j] K[j]
//   dK[j]   = scale sum_i dS[i,j] Q[i]      (summed over the GQA group's heads)
//   dV[j]   =       sum_i P[i,j] dO[i]      (likewise)
// (delta_i = sum_j P[i,j] dP[i,j], the softmax Jacobian's row term.)
//
// Two kernels share the forward's machinery (TMA tiles with 128-byte swizzle,
// tcgen05 MMAs with fp32 accumulators in tensor memory, one thread per
// 128-lane row), each with 320 threads: warps 0-7 do the elementwise work and
// the epilogue (two per SM sub-partition, each on half a tile's columns), warp
// 8 is the TMA producer, warp 9 issues the MMAs.
//   dQ kernel:  work item (b, h, 128-row query tile), walking the key tiles
//               the tile sees: S = Q K^T and dP = dO V^T into tensor memory,
//               dS (bf16) written over dP, then dQ += dS K.
//   dKV kernel: work item (b, KV head, 128-key tile), walking the query tiles
//               of every head of the group that see it: S^T = K Q^T and
//               dP^T = V dO^T, P^T and dS^T (bf16) both written over dP^T,
//               then dV += P^T dO and dK += dS^T Q; S^T of the next query
//               tile is computed while the exponentials of this one run.
#pragma once

#include <cuda_bf16.h>
#include <math_constants.h>

#include "tfa_plan.h"
#include "tfa_ptx.cuh"

namespace tfa {
namespace bwd {

// Warps 0-7: elementwise (warp w holds tensor-memory lanes 32 (w % 4) ..,
// i.e. 32 rows, and half w / 4 of each tile's 128 columns: two warps per SM
// sub-partition); warp 8: TMA producer; warp 9: MMA issuer.
constexpr int kEwWarps = 8;
constexpr int kThreads = 32 * (kEwWarps + 2);

template <int D>
struct Cfg {
    static_assert(D == 64 || D == 128, "head dim");
    static constexpr int kTileBytes = 128 * D * 2;
    static constexpr int kColBlocks = D / 64;
    static constexpr int kColBlockBytes = 128 * 128;
    static constexpr int kSlots = (D == 128) ? 4 : 8;  // ring of streamed tiles
    static constexpr int kFixOff = 0;                  // two tiles fixed per item
    static constexpr int kRingOff = 2 * kTileBytes;
    static constexpr int kBarOff = kRingOff + kSlots * kTileBytes;
    static constexpr int kNumBars = 2 * kSlots + 11;
    static constexpr int kMiscOff = kBarOff + kNumBars * 8;
    // dKV kernel: per elementwise warp, the step's 128 values of -lse and delta
    static constexpr int kStageOff = kMiscOff + 16;
    static constexpr int kSmemBytes = kStageOff + kEwWarps * 256 * 4 + 1024;  // + slack to align the base
    static constexpr uint32_t kTmemCols = 512;
    static constexpr uint32_t kTmemA = 0;    // S (dQ kernel) / S^T (dKV kernel), 128 columns
    static constexpr uint32_t kTmemB = 128;  // dP / dP^T, 128 columns
    static constexpr uint32_t kTmemC = 256;  // dQ accumulator / dV accumulator, D columns
    static constexpr uint32_t kTmemD = 256 + D;  // dK accumulator (dKV kernel), D columns
    static constexpr uint32_t kTmemA2 = 256 + D;  // dQ kernel: second S buffer (odd key tiles), 128 columns
};

struct BwdParams {
    __nv_bfloat16 *dq, *dk, *dv;  // outputs: [B,Hq,L,D], [B,Hkv,S,D] x2
    const float *lse, *delta;     // [B,Hq,L]
    const float *key_mask;        // [B,S] or nullptr
    unsigned *status;
    int B, Hq, Hkv, L, S, G, causal, window;
    float scale, scale_log2;
    int n_items;
};

// Barriers: fixed tiles full/empty, ring full/empty, the two score matrices
// ready, the bf16 operands written, accumulators ready / read, teardown.
struct Bars {
    uint32_t base;
    int slots;
    __device__ __forceinline__ uint32_t fix_full() const { return base; }
    __device__ __forceinline__ uint32_t fix_empty() const { return base + 8; }
    __device__ __forceinline__ uint32_t ring_full(int s) const { return base + 8 * (2 + s); }
    __device__ __forceinline__ uint32_t ring_empty(int s) const { return base + 8 * (2 + slots + s); }
    __device__ __forceinline__ uint32_t mm_full() const { return base + 8 * (2 + 2 * slots); }
    __device__ __forceinline__ uint32_t op_full() const { return base + 8 * (3 + 2 * slots); }
    __device__ __forceinline__ uint32_t acc_full() const { return base + 8 * (4 + 2 * slots); }
    __device__ __forceinline__ uint32_t acc_empty() const { return base + 8 * (5 + 2 * slots); }
    __device__ __forceinline__ uint32_t done() const { return base + 8 * (6 + 2 * slots); }
    // dKV kernel, two phases per step: dP^T ready (mm_full: S^T ready), and
    // P^T written (op_full: dS^T written)
    __device__ __forceinline__ uint32_t dp_full() const { return base + 8 * (7 + 2 * slots); }
    __device__ __forceinline__ uint32_t pt_full() const { return base + 8 * (8 + 2 * slots); }
    // dQ kernel: S of odd key tiles (its second buffer; mm_full: even ones).
    // One barrier per buffer: S_{x+2} is issued only after S_x was consumed,
    // so neither runs two phases ahead of its waiter.
    __device__ __forceinline__ uint32_t s2_full() const { return base + 8 * (9 + 2 * slots); }
    // dKV kernel: every elementwise warp has read S^T_i (S^T_{i+1} may overwrite it)
    __device__ __forceinline__ uint32_t s_free() const { return base + 8 * (10 + 2 * slots); }
};

// delta_i = sum_d dO[i,d] O[i,d] (fp32), one warp per row.
template <int D>
__global__ void __launch_bounds__(256) delta_kernel(const __nv_bfloat16 *o, const __nv_bfloat16 *dout,
                                                    float *delta, long long rows) {
    const long long row = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    constexpr int kPer = D / 32;  // elements per lane: 4 (D = 128) or 2 (D = 64)
    const __nv_bfloat16 *po = o + row * D + lane * kPer;
    const __nv_bfloat16 *pd = dout + row * D + lane * kPer;
    float acc = 0.f;
#pragma unroll
    for (int e = 0; e < kPer; e += 2) {
        const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(po + e));
        const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(pd + e));
        acc = fmaf(a.x, b.x, fmaf(a.y, b.y, acc));
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (lane == 0) delta[row] = acc;
}

// Item enumeration shared by the roles of one CTA.  Items are numbered in
// roughly descending order of work -- dQ kernel: item = (qt, b, h), query tiles
// in descending order when causal (longest key ranges first); dKV kernel:
// item = (kt, b, g), key tiles ascending (when causal, later key tiles are
// seen by fewer query tiles) -- and dealt in snake order: CTA c takes items
// c, 2G-1-c, 2G+c, 4G-1-c, ... (G CTAs), so one round's largest items go
// with the next round's smallest and the CTAs' totals even out.
struct ItemIter {
    int item, stride;
    __device__ __forceinline__ ItemIter()
        : item(static_cast<int>(blockIdx.x)), stride(2 * static_cast<int>(gridDim.x) - 1 - 2 * item) {}
    __device__ __forceinline__ void next() {
        item += stride;
        stride = 2 * static_cast<int>(gridDim.x) - stride;
    }
};
struct QItem {
    int b, h, qt, lo, hi;  // key tiles [lo, hi]
};
__device__ __forceinline__ QItem q_item(const BwdParams &p, int item) {
    const int nqt = (p.L + kBlockQ - 1) / kBlockQ;
    const int bh = p.B * p.Hq;
    const int r = item / bh, rem = item - r * bh;
    QItem it;
    it.qt = p.causal ? nqt - 1 - r : r;
    it.b = rem / p.Hq;
    it.h = rem - it.b * p.Hq;
    const KeyRange kr = qtile_key_range(p.L, p.S, p.causal, p.window, it.qt * kBlockQ, 0u);
    it.lo = kr.lo;
    it.hi = kr.hi;
    return it;
}
struct KItem {
    int b, g, kt, qlo, qhi, nq, steps;  // per head of the group: query tiles [qlo, qhi]
};
__device__ __forceinline__ KItem k_item(const BwdParams &p, int item) {
    const int bg = p.B * p.Hkv;
    const int kt = item / bg, rem = item - kt * bg;
    KItem it;
    it.kt = kt;
    it.b = rem / p.Hkv;
    it.g = rem - it.b * p.Hkv;
    const KeyRange qr = ktile_query_range(p.L, p.S, p.causal, p.window, kt);
    it.qlo = qr.lo;
    it.qhi = qr.hi;
    it.nq = qr.hi >= qr.lo ? qr.hi - qr.lo + 1 : 0;
    it.steps = it.nq * p.G;
    return it;
}

// Common set-up of both kernels: barriers, tensor memory, the abort flag.
template <int D>
struct Setup {
    uint32_t sbase, tmem;
    uint8_t *gbase;
    Bars bar;
    volatile int *abort_flag;
};

template <int D>
__device__ __forceinline__ Setup<D> setup(const CUtensorMap *m0, const CUtensorMap *m1,
                                          const CUtensorMap *m2, const CUtensorMap *m3) {
    using C = Cfg<D>;
    extern __shared__ uint8_t smem_raw[];
    Setup<D> st;
    const uint32_t raw = smem_addr(smem_raw);
    st.sbase = (raw + 1023u) & ~1023u;
    st.gbase = smem_raw + (st.sbase - raw);
    st.bar = Bars{st.sbase + C::kBarOff, C::kSlots};
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(st.gbase + C::kMiscOff);
    st.abort_flag = reinterpret_cast<volatile int *>(st.gbase + C::kMiscOff + 4);
    const int warp = threadIdx.x >> 5;
    if (threadIdx.x == 0) {
        mbar_init(st.bar.fix_full(), 1);
        mbar_init(st.bar.fix_empty(), 1);
        for (int s = 0; s < C::kSlots; ++s) {
            mbar_init(st.bar.ring_full(s), 1);
            mbar_init(st.bar.ring_empty(s), 1);
        }
        mbar_init(st.bar.mm_full(), 1);
        mbar_init(st.bar.op_full(), kEwWarps);
        mbar_init(st.bar.acc_full(), 1);
        mbar_init(st.bar.acc_empty(), kEwWarps);
        mbar_init(st.bar.done(), 1);
        mbar_init(st.bar.dp_full(), 1);
        mbar_init(st.bar.pt_full(), kEwWarps);
        mbar_init(st.bar.s2_full(), 1);
        mbar_init(st.bar.s_free(), kEwWarps);
        *st.abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(smem_addr(tmem_slot), C::kTmemCols);
        tmem_relinquish();
    }
    if (warp == kEwWarps && (threadIdx.x & 31) == 0) {
        prefetch_tensormap(m0);
        prefetch_tensormap(m1);
        prefetch_tensormap(m2);
        prefetch_tensormap(m3);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    st.tmem = *tmem_slot;
    return st;
}

template <int D>
__device__ __forceinline__ void teardown(const Setup<D> &st) {
    tc_fence_before();
    __syncthreads();
    if ((threadIdx.x >> 5) == 0) {
        tc_fence_after();
        tmem_dealloc(st.tmem, Cfg<D>::kTmemCols);
    }
}

// The producer's exit: every copy it started must land before the CTA leaves.
template <int D>
__device__ __forceinline__ void drain_copies(const Bars &bar, uint32_t prod, uint32_t fix_use) {
    using C = Cfg<D>;
    for (uint32_t s = 0; s < (uint32_t)C::kSlots; ++s) {
        if (prod > s) {
            const uint32_t armed = (prod - s - 1) / C::kSlots + 1;
            mbar_drain(bar.ring_full(s), (armed - 1) & 1);
        }
    }
    if (fix_use > 0) mbar_drain(bar.fix_full(), (fix_use - 1) & 1);
}

// Load two [128 rows][D] tiles (64-column boxes) onto one barrier.
template <int D>
__device__ __forceinline__ void load_tile(uint32_t dst, const CUtensorMap *map, uint32_t bar, int row,
                                          int plane) {
    using C = Cfg<D>;
    for (int cb = 0; cb < C::kColBlocks; ++cb)
        tma_load_3d(dst + cb * C::kColBlockBytes, map, bar, cb * 64, row, plane);
}

// Tensor-memory column of K-step kk (16 keys or queries, 8 packed bf16x2
// columns) of an operand the elementwise warps wrote: half h of the 128
// columns writes its 32 packed columns at 64 h, over columns it has read.
__device__ __forceinline__ uint32_t packed_col(int kk) { return kk * 8 + (kk >= 4 ? 32 : 0); }

// K-step offset (>> 4) inside a K-major 128-byte-swizzled [128][D] tile.
template <int D>
__device__ __forceinline__ uint32_t kstep_off(int kk) {
    return static_cast<uint32_t>(((kk >> 2) * Cfg<D>::kColBlockBytes + (kk & 3) * 32) >> 4);
}

// dKV kernel ring: slots in pairs, step n (counted over the CTA's items) uses
// pair n % kPairs and alternates which of the two holds Q and which dO, so
// Q_n takes the slot dO_{n - kPairs} left.  dO is released after dV, a phase
// before Q is released after dK, so Q (needed first: S^T_n is issued while
// step n-1's elementwise work runs) lands a phase earlier than in a plain
// ring.  Each slot is used once per kPairs steps: use index n / kPairs.
template <int D>
struct KvRing {  // dQ kernel: q_slot holds K_t, do_slot V_t
    static constexpr uint32_t kPairs = Cfg<D>::kSlots / 2;
    __device__ __forceinline__ static uint32_t q_slot(uint32_t n) { return 2 * (n % kPairs) + ((n / kPairs) & 1); }
    __device__ __forceinline__ static uint32_t do_slot(uint32_t n) {
        return 2 * (n % kPairs) + (((n / kPairs) & 1) ^ 1);
    }
    __device__ __forceinline__ static uint32_t use(uint32_t n) { return n / kPairs; }
};

// ------------------------------------------------------------------ dQ kernel
template <int D, bool KM>
__global__ void __launch_bounds__(kThreads, 1)
    dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
              const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
              const BwdParams p) {
    using C = Cfg<D>;
    const Setup<D> st = setup<D>(&tm_q, &tm_do, &tm_k, &tm_v);
    // The dK/dV kernel reads none of this kernel's output: it may take over
    // each SM as soon as this kernel's CTA there retires.
    if (threadIdx.x == 0) grid_dep_launch();
    const Bars &bar = st.bar;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr uint32_t kTileStep = C::kTileBytes >> 4;

    if (warp == kEwWarps) {
        // ---- producer: Q and dO once per item, then K_j, V_j per key tile
        if (lane == 0) {
            using R = KvRing<D>;
            uint32_t t = 0, fix_use = 0;
            uint32_t used[C::kSlots];
#pragma unroll
            for (int s = 0; s < C::kSlots; ++s) used[s] = 0;
            for (ItemIter ii; ii.item < p.n_items; ii.next()) {
                const QItem it = q_item(p, ii.item);
                if (fix_use > 0 && !mbar_wait(bar.fix_empty(), (fix_use - 1) & 1, st.abort_flag, p.status))
                    break;
                mbar_arrive_expect_tx(bar.fix_full(), 2 * C::kTileBytes);
                load_tile<D>(st.sbase + C::kFixOff, &tm_q, bar.fix_full(), it.qt * kBlockQ, it.b * p.Hq + it.h);
                load_tile<D>(st.sbase + C::kFixOff + C::kTileBytes, &tm_do, bar.fix_full(), it.qt * kBlockQ,
                             it.b * p.Hq + it.h);
                ++fix_use;
                bool stop = false;
                for (int j = it.lo; j <= it.hi && !stop; ++j, ++t) {
                    const uint32_t u = R::use(t);
                    for (int which = 0; which < 2; ++which) {  // K_t then V_t
                        const uint32_t s = which ? R::do_slot(t) : R::q_slot(t);
                        if (u > 0 && !mbar_wait(bar.ring_empty(s), (u - 1) & 1, st.abort_flag, p.status)) {
                            stop = true;
                            break;
                        }
                        mbar_arrive_expect_tx(bar.ring_full(s), C::kTileBytes);
                        load_tile<D>(st.sbase + C::kRingOff + s * C::kTileBytes, which ? &tm_v : &tm_k,
                                     bar.ring_full(s), j * kBlockK, it.b * p.Hkv + it.h / p.G);
                        ++used[s];
                    }
                }
                if (stop) break;
            }
            for (int s = 0; s < C::kSlots; ++s)
                if (used[s] > 0) mbar_drain(bar.ring_full(s), (used[s] - 1) & 1);
            if (fix_use > 0) mbar_drain(bar.fix_full(), (fix_use - 1) & 1);
        }
    } else if (warp == kEwWarps + 1) {
        // ---- MMA issuer
        if (lane == 0) {
            constexpr uint32_t kIdescS = idesc_bf16_f32(128, kBlockK, 0);  // both operands K-major
            constexpr uint32_t kIdescDQ = idesc_bf16_f32(128, D, 1);       // B = K tile, MN-major
            const uint64_t d_q = smem_desc_sw128(st.sbase + C::kFixOff, 16, 1024);
            const uint64_t d_do = d_q + kTileStep;
            const uint64_t d_ring = smem_desc_sw128(st.sbase + C::kRingOff, 16, 1024);
            const uint64_t d_ring_mn = smem_desc_sw128(st.sbase + C::kRingOff, C::kColBlockBytes, 1024);
            using R = KvRing<D>;
            uint32_t tb = 0, fix_use = 0, op_cnt = 0, acc_use = 0;
            for (ItemIter ii; ii.item < p.n_items; ii.next()) {
                const QItem it = q_item(p, ii.item);
                if (!mbar_wait(bar.fix_full(), fix_use & 1, st.abort_flag, p.status)) goto mma_out;
                ++fix_use;
                // S_j alternates between two buffers and runs two key tiles
                // ahead of dQ; dP_{j+1} follows dQ += dS_j K_j (dS_j lies over dP_j's
                // columns).  The elementwise warps compute P_{j+1} from S_{j+1} while
                // the tensor core finishes step j.
                const int n = it.hi - it.lo + 1;
                // K_t and V_t of the CTA's t-th key tile (counted over its items)
                auto take = [&](uint32_t &slot, uint32_t t, int which) -> bool {
                    slot = which ? R::do_slot(t) : R::q_slot(t);
                    return mbar_wait(bar.ring_full(slot), R::use(t) & 1, st.abort_flag, p.status);
                };
                auto issue_s = [&](int x, uint32_t ks) {
                    const uint32_t dst = st.tmem + ((x & 1) ? C::kTmemA2 : C::kTmemA);
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk)
                        umma_ss(dst, d_q + kstep_off<D>(kk), d_ring + ks * kTileStep + kstep_off<D>(kk), kIdescS,
                                kk > 0 ? 1u : 0u);
                    umma_commit((x & 1) ? bar.s2_full() : bar.mm_full());
                };
                auto issue_dp = [&](uint32_t vs) {
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk)
                        umma_ss(st.tmem + C::kTmemB, d_do + kstep_off<D>(kk), d_ring + vs * kTileStep + kstep_off<D>(kk),
                                kIdescS, kk > 0 ? 1u : 0u);
                    umma_commit(bar.dp_full());
                    umma_commit(bar.ring_empty(vs));  // V's only use
                };
                uint32_t k_cur = 0, k_nxt = 0, v_nxt = 0, v0 = 0;
                if (!take(k_cur, tb, 0) || !take(v0, tb, 1)) goto mma_out;
                tc_fence_after();
                issue_s(0, k_cur);
                issue_dp(v0);
                if (n > 1) {
                    if (!take(k_nxt, tb + 1, 0) || !take(v_nxt, tb + 1, 1)) goto mma_out;
                    tc_fence_after();
                    issue_s(1, k_nxt);
                }
                if (n == 1) umma_commit(bar.fix_empty());  // Q, dO's last use
                for (int x = 0; x < n; ++x) {
                    // dQ += dS K, dS (bf16) over dP columns 0-31 and 64-95
                    if (!mbar_wait(bar.op_full(), op_cnt & 1, st.abort_flag, p.status)) goto mma_out;
                    ++op_cnt;
                    // the previous item's dQ must have been read before it is overwritten
                    if (x == 0 && acc_use > 0 &&
                        !mbar_wait(bar.acc_empty(), (acc_use - 1) & 1, st.abort_flag, p.status))
                        goto mma_out;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < kBlockK / 16; ++kk)
                        umma_ts(st.tmem + C::kTmemC, st.tmem + C::kTmemB + packed_col(kk),
                                d_ring_mn + k_cur * kTileStep + kk * ((16 * 128) >> 4), kIdescDQ,
                                (x > 0 || kk > 0) ? 1u : 0u);
                    umma_commit(bar.ring_empty(k_cur));  // K_j's last use
                    if (x + 1 < n) {
                        issue_dp(v_nxt);
                        if (x + 2 == n) umma_commit(bar.fix_empty());  // Q, dO's last use
                    }
                    uint32_t k_nn = 0, v_nn = 0;
                    if (x + 2 < n) {
                        if (!take(k_nn, tb + x + 2, 0) || !take(v_nn, tb + x + 2, 1)) goto mma_out;
                        tc_fence_after();
                        issue_s(x + 2, k_nn);
                    }
                    k_cur = k_nxt;
                    k_nxt = k_nn;
                    v_nxt = v_nn;
                }
                umma_commit(bar.acc_full());
                ++acc_use;
                tb += static_cast<uint32_t>(n);
            }
        mma_out:
            umma_commit(bar.done());
            mbar_drain(bar.done(), 0);
        }
    } else {
        // ---- elementwise (warps 0-7): P, dS per key tile; dQ epilogue per item
        const int r = (warp & 3) * 32 + lane;  // query row inside the tile = tensor-memory lane
        const int hf = warp >> 2;               // key columns 64 hf .. 64 hf + 63
        const uint32_t lane_base = (static_cast<uint32_t>(warp & 3) * 32u) << 16;
        const uint32_t tA = st.tmem + C::kTmemA + lane_base;
        const uint32_t tA2 = st.tmem + C::kTmemA2 + lane_base;
        const uint32_t tB = st.tmem + C::kTmemB + lane_base;
        const uint32_t tC = st.tmem + C::kTmemC + lane_base;
        const float c = p.scale_log2;
        uint32_t mm_cnt = 0, acc_cnt = 0;  // mm_cnt: dP tiles seen
        uint32_t s_even = 0, s_odd = 0;    // S tiles seen per buffer
        for (ItemIter ii; ii.item < p.n_items; ii.next()) {
            const QItem it = q_item(p, ii.item);
            const int q0 = it.qt * kBlockQ;
            const int row = q0 + r;
            const bool valid = row < p.L;
            const size_t idx = static_cast<size_t>(it.b * p.Hq + it.h) * p.L + row;
            const float lse_r = valid ? __ldg(p.lse + idx) : CUDART_INF_F;
            const float dl_r = valid ? __ldg(p.delta + idx) : 0.f;
            const int pos = (p.S - p.L) + row;
            const int hi_abs = p.causal ? imin(pos, p.S - 1) : p.S - 1;
            const int lo_abs = (p.causal && p.window > 0) ? pos - p.window + 1 : 0;
            const float *km_row = KM ? p.key_mask + static_cast<size_t>(it.b) * p.S : nullptr;
            for (int j = it.lo; j <= it.hi; ++j) {
                // phase 1: P = 2^(S c - lse) from S (its buffer alternates per key tile)
                const bool odd = ((j - it.lo) & 1) != 0;
                const uint32_t sph = (odd ? s_odd++ : s_even++) & 1;
                if (!__all_sync(0xffffffffu, mbar_wait(odd ? bar.s2_full() : bar.mm_full(), sph, st.abort_flag, p.status)))
                    goto ew_out;
                tc_fence_after();
                const uint32_t tS = odd ? tA2 : tA;
                const bool needs = key_tile_needs_mask(p.L, p.S, p.causal, p.window, KM ? 1 : 0, q0, j, 0u);
                float pr[64];
#pragma unroll
                for (int c2 = 0; c2 < 2; ++c2) {
                    const int ch = 2 * hf + c2;
                    uint32_t sv[32];
                    tmem_ld32(tS + 32 * ch, sv);
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        float pe = ex2(fmaf(__uint_as_float(sv[e]), c, -lse_r));
                        if (needs) {
                            const int k = j * kBlockK + 32 * ch + e;
                            const bool al = k >= lo_abs && k <= hi_abs && (!KM || __ldg(km_row + k) > 0.5f);
                            pe = al ? pe : 0.f;
                        }
                        pr[32 * c2 + e] = pe;
                    }
                }
                // phase 2: dS = P (dP - delta) from dP, over dP's columns
                if (!__all_sync(0xffffffffu, mbar_wait(bar.dp_full(), mm_cnt & 1, st.abort_flag, p.status)))
                    goto ew_out;
                ++mm_cnt;
                tc_fence_after();
#pragma unroll
                for (int c2 = 0; c2 < 2; ++c2) {
                    const int ch = 2 * hf + c2;
                    uint32_t dv[32], w[16];
                    tmem_ld32(tB + 32 * ch, dv);
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        w[e] = pack_bf16(pr[32 * c2 + 2 * e] * (__uint_as_float(dv[2 * e]) - dl_r),
                                         pr[32 * c2 + 2 * e + 1] * (__uint_as_float(dv[2 * e + 1]) - dl_r));
                    tmem_st16(tB + 64 * hf + 16 * c2, w);  // over dP columns this warp has read
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar.op_full());
            }
            if (!__all_sync(0xffffffffu, mbar_wait(bar.acc_full(), acc_cnt & 1, st.abort_flag, p.status)))
                goto ew_out;
            ++acc_cnt;
            tc_fence_after();
            {
                __nv_bfloat16 *orow = valid ? p.dq + idx * D : nullptr;
#pragma unroll
                for (int cc = hf * (D / 64); cc < (hf + 1) * (D / 64); ++cc) {
                    uint32_t o[32];
                    tmem_ld32(tC + 32 * cc, o);
                    uint32_t w[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        w[i] = pack_bf16(__uint_as_float(o[2 * i]) * p.scale, __uint_as_float(o[2 * i + 1]) * p.scale);
                    if (orow) {
                        uint4 *dst = reinterpret_cast<uint4 *>(orow + cc * 32);
#pragma unroll
                        for (int v4 = 0; v4 < 4; ++v4)
                            dst[v4] = make_uint4(w[4 * v4], w[4 * v4 + 1], w[4 * v4 + 2], w[4 * v4 + 3]);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar.acc_empty());
        }
    ew_out:;
    }
    teardown<D>(st);
}

// ----------------------------------------------------------------- dKV kernel
template <int D, bool KM>
__global__ void __launch_bounds__(kThreads, 1)
    dkv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
               const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
               const BwdParams p) {
    using C = Cfg<D>;
    const Setup<D> st = setup<D>(&tm_q, &tm_do, &tm_k, &tm_v);
    const Bars &bar = st.bar;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr uint32_t kTileStep = C::kTileBytes >> 4;

    if (warp == kEwWarps) {
        // ---- producer: K and V once per item, then Q_i, dO_i per (head, query tile)
        if (lane == 0) {
            using R = KvRing<D>;
            uint32_t n = 0, fix_use = 0;
            uint32_t used[C::kSlots];
#pragma unroll
            for (int s = 0; s < C::kSlots; ++s) used[s] = 0;
            bool stop = false;
            for (ItemIter ii; ii.item < p.n_items && !stop; ii.next()) {
                const KItem it = k_item(p, ii.item);
                if (it.steps == 0) continue;
                if (fix_use > 0 && !mbar_wait(bar.fix_empty(), (fix_use - 1) & 1, st.abort_flag, p.status))
                    break;
                mbar_arrive_expect_tx(bar.fix_full(), 2 * C::kTileBytes);
                load_tile<D>(st.sbase + C::kFixOff, &tm_k, bar.fix_full(), it.kt * kBlockK, it.b * p.Hkv + it.g);
                load_tile<D>(st.sbase + C::kFixOff + C::kTileBytes, &tm_v, bar.fix_full(), it.kt * kBlockK,
                             it.b * p.Hkv + it.g);
                ++fix_use;
                for (int step = 0; step < it.steps && !stop; ++step, ++n) {
                    const int h = it.g * p.G + step / it.nq;
                    const int qt = it.qlo + step % it.nq;
                    const uint32_t u = R::use(n);
                    for (int which = 0; which < 2; ++which) {  // Q_n then dO_n
                        const uint32_t s = which ? R::do_slot(n) : R::q_slot(n);
                        if (u > 0 && !mbar_wait(bar.ring_empty(s), (u - 1) & 1, st.abort_flag, p.status)) {
                            stop = true;
                            break;
                        }
                        mbar_arrive_expect_tx(bar.ring_full(s), C::kTileBytes);
                        load_tile<D>(st.sbase + C::kRingOff + s * C::kTileBytes, which ? &tm_do : &tm_q,
                                     bar.ring_full(s), qt * kBlockQ, it.b * p.Hq + h);
                        ++used[s];
                    }
                }
            }
            // every copy started must land before the CTA leaves
            for (int s = 0; s < C::kSlots; ++s)
                if (used[s] > 0) mbar_drain(bar.ring_full(s), (used[s] - 1) & 1);
            if (fix_use > 0) mbar_drain(bar.fix_full(), (fix_use - 1) & 1);
        }
    } else if (warp == kEwWarps + 1) {
        // ---- MMA issuer
        if (lane == 0) {
            constexpr uint32_t kIdescS = idesc_bf16_f32(128, kBlockQ, 0);  // both operands K-major
            constexpr uint32_t kIdescAcc = idesc_bf16_f32(128, D, 1);      // B = dO / Q tile, MN-major
            const uint64_t d_k = smem_desc_sw128(st.sbase + C::kFixOff, 16, 1024);
            const uint64_t d_v = d_k + kTileStep;
            const uint64_t d_ring = smem_desc_sw128(st.sbase + C::kRingOff, 16, 1024);
            const uint64_t d_ring_mn = smem_desc_sw128(st.sbase + C::kRingOff, C::kColBlockBytes, 1024);
            using R = KvRing<D>;
            uint32_t n = 0, fix_use = 0, sf_cnt = 0, op_cnt = 0, acc_use = 0;
            for (ItemIter ii; ii.item < p.n_items; ii.next()) {
                const KItem it = k_item(p, ii.item);
                if (it.steps == 0) continue;
                if (!mbar_wait(bar.fix_full(), fix_use & 1, st.abort_flag, p.status)) goto mma_out;
                ++fix_use;
                // Per step i: S^T_{i+1} as soon as the elementwise warps have read
                // S^T_i; dV += P^T_i dO_i once P^T_i is written; dK += dS^T_i Q_i
                // once dS^T_i is written, then dP^T_{i+1}.  P^T_i and dS^T_i (bf16)
                // lie over dP^T_i's columns (packed columns 0-31 / 64-95 and 32-63 /
                // 96-127), so S^T's columns are free as soon as they are read and
                // S^T_{i+1} overlaps the exponentials of step i.
                auto take = [&](uint32_t slot, uint32_t m) -> bool {
                    return mbar_wait(bar.ring_full(slot), R::use(m) & 1, st.abort_flag, p.status);
                };
                auto issue_st = [&](uint32_t m) {  // S^T = K Q_m^T
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk)
                        umma_ss(st.tmem + C::kTmemA, d_k + kstep_off<D>(kk),
                                d_ring + R::q_slot(m) * kTileStep + kstep_off<D>(kk), kIdescS, kk > 0 ? 1u : 0u);
                    umma_commit(bar.mm_full());
                };
                auto issue_dpt = [&](uint32_t m) {  // dP^T = V dO_m^T
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk)
                        umma_ss(st.tmem + C::kTmemB, d_v + kstep_off<D>(kk),
                                d_ring + R::do_slot(m) * kTileStep + kstep_off<D>(kk), kIdescS, kk > 0 ? 1u : 0u);
                    umma_commit(bar.dp_full());
                };
                if (!take(R::q_slot(n), n) || !take(R::do_slot(n), n)) goto mma_out;
                tc_fence_after();
                issue_st(n);
                issue_dpt(n);
                if (it.steps == 1) umma_commit(bar.fix_empty());
                for (int step = 0; step < it.steps; ++step) {
                    const uint32_t cur = n + step;
                    const bool more = step + 1 < it.steps;
                    if (more) {
                        if (!mbar_wait(bar.s_free(), sf_cnt & 1, st.abort_flag, p.status)) goto mma_out;
                        ++sf_cnt;
                        if (!take(R::q_slot(cur + 1), cur + 1)) goto mma_out;
                        tc_fence_after();
                        issue_st(cur + 1);
                    }
                    // the previous item's dK, dV must have been read before they restart
                    if (step == 0 && acc_use > 0 &&
                        !mbar_wait(bar.acc_empty(), (acc_use - 1) & 1, st.abort_flag, p.status))
                        goto mma_out;
                    // dV += P^T dO, dK += dS^T Q and dP^T_{i+1} as one run of MMAs once
                    // both operands are written: every wait of the issuer between
                    // MMA blocks lets the tensor pipe drain
                    if (!mbar_wait(bar.op_full(), op_cnt & 1, st.abort_flag, p.status)) goto mma_out;
                    ++op_cnt;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < kBlockQ / 16; ++kk)
                        umma_ts(st.tmem + C::kTmemC, st.tmem + C::kTmemB + packed_col(kk),
                                d_ring_mn + R::do_slot(cur) * kTileStep + kk * ((16 * 128) >> 4), kIdescAcc,
                                (step > 0 || kk > 0) ? 1u : 0u);
                    umma_commit(bar.ring_empty(R::do_slot(cur)));  // dO_i's last use
#pragma unroll
                    for (int kk = 0; kk < kBlockQ / 16; ++kk)
                        umma_ts(st.tmem + C::kTmemD, st.tmem + C::kTmemB + 32 + packed_col(kk),
                                d_ring_mn + R::q_slot(cur) * kTileStep + kk * ((16 * 128) >> 4), kIdescAcc,
                                (step > 0 || kk > 0) ? 1u : 0u);
                    umma_commit(bar.ring_empty(R::q_slot(cur)));  // Q_i's last use
                    if (more) {  // dP^T_{i+1} over the columns dV, dK have just read
                        if (!take(R::do_slot(cur + 1), cur + 1)) goto mma_out;
                        tc_fence_after();
                        issue_dpt(cur + 1);
                        if (step + 2 == it.steps) umma_commit(bar.fix_empty());  // K, V's last use
                    }
                }
                umma_commit(bar.acc_full());
                ++acc_use;
                n += it.steps;
            }
        mma_out:
            umma_commit(bar.done());
            mbar_drain(bar.done(), 0);
        }
    } else {
        // ---- elementwise (warps 0-7): P^T, dS^T per step; dK, dV epilogue per item
        const int r = (warp & 3) * 32 + lane;  // key row inside the tile = tensor-memory lane
        const int hf = warp >> 2;               // query columns 64 hf .. 64 hf + 63
        const uint32_t lane_base = (static_cast<uint32_t>(warp & 3) * 32u) << 16;
        const uint32_t tA = st.tmem + C::kTmemA + lane_base;
        const uint32_t tB = st.tmem + C::kTmemB + lane_base;
        const uint32_t tC = st.tmem + C::kTmemC + lane_base;
        const uint32_t tD = st.tmem + C::kTmemD + lane_base;
        const float c = p.scale_log2;
        const int P = p.S - p.L;
        float *stage = reinterpret_cast<float *>(st.gbase + C::kStageOff) + warp * 256;
        uint32_t mm_cnt = 0, acc_cnt = 0;
        for (ItemIter ii; ii.item < p.n_items; ii.next()) {
            const KItem it = k_item(p, ii.item);
            const int key = it.kt * kBlockK + r;
            const bool kvalid = key < p.S;
            const bool kept = kvalid && (!KM || __ldg(p.key_mask + static_cast<size_t>(it.b) * p.S + key) > 0.5f);
            // the query rows that see this key: [q_lo, q_hi] (empty when not kept)
            int q_lo = p.causal ? imax(0, key - P) : 0;
            int q_hi = (p.causal && p.window > 0) ? imin(p.L - 1, key - P + p.window - 1) : p.L - 1;
            if (!kept) q_hi = q_lo - 1;
            const size_t oidx = (static_cast<size_t>(it.b * p.Hkv + it.g) * p.S + key) * D;
            if (it.steps == 0) {  // no row sees this key tile: zero gradients
                if (kvalid) {
                    uint4 *dk4 = reinterpret_cast<uint4 *>(p.dk + oidx);
                    uint4 *dv4 = reinterpret_cast<uint4 *>(p.dv + oidx);
                    for (int v4 = hf * (D / 16); v4 < (hf + 1) * (D / 16); ++v4) {
                        dk4[v4] = make_uint4(0u, 0u, 0u, 0u);
                        dv4[v4] = make_uint4(0u, 0u, 0u, 0u);
                    }
                }
                continue;
            }
            // -lse and delta of the warp's 64 query columns of step i (lane e:
            // columns 32 c2 + e of its half), fetched one step ahead into
            // registers, written to the warp's stage at the step's start and
            // read back as shared-memory broadcasts
            float nxt[4];
            auto fetch = [&](int step) {
                const int h = it.g * p.G + step / it.nq;
                const int q0 = (it.qlo + step % it.nq) * kBlockQ;
                const float *lse_h = p.lse + static_cast<size_t>(it.b * p.Hq + h) * p.L;
                const float *dl_h = p.delta + static_cast<size_t>(it.b * p.Hq + h) * p.L;
#pragma unroll
                for (int c2 = 0; c2 < 2; ++c2) {
                    const int q = q0 + 64 * hf + 32 * c2 + lane;
                    nxt[2 * c2] = q < p.L ? -__ldg(lse_h + q) : -CUDART_INF_F;
                    nxt[2 * c2 + 1] = q < p.L ? __ldg(dl_h + q) : 0.f;
                }
            };
            fetch(0);
            for (int step = 0; step < it.steps; ++step) {
                const bool more = step + 1 < it.steps;
                const int q0 = (it.qlo + step % it.nq) * kBlockQ + 64 * hf;  // the warp's first query column
                __syncwarp();  // every lane is done with the previous step's stage
#pragma unroll
                for (int c2 = 0; c2 < 2; ++c2) {
                    stage[64 * hf + 32 * c2 + lane] = nxt[2 * c2];
                    stage[128 + 64 * hf + 32 * c2 + lane] = nxt[2 * c2 + 1];
                }
                __syncwarp();
                // S^T_i: read it, then free its columns for S^T_{i+1}
                if (!__all_sync(0xffffffffu, mbar_wait(bar.mm_full(), mm_cnt & 1, st.abort_flag, p.status)))
                    goto ew_out;
                tc_fence_after();
                uint32_t sv[64];
                tmem_ld64(tA + 64 * hf, sv);
                if (more) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bar.s_free());
                    fetch(step + 1);
                }
                // P^T = 2^(S^T c - lse), kept in fp32 for dS^T
                float pt[64];
#pragma unroll
                for (int e = 0; e < 64; ++e) {
                    const bool allowed = (q0 + e >= q_lo) & (q0 + e <= q_hi);
                    const float ev = ex2(fmaf(__uint_as_float(sv[e]), c, stage[64 * hf + e]));
                    pt[e] = allowed ? ev : 0.f;
                }
                // dP^T_i: its first 32 columns of the half, then P^T (bf16) over them
                if (!__all_sync(0xffffffffu, mbar_wait(bar.dp_full(), mm_cnt & 1, st.abort_flag, p.status)))
                    goto ew_out;
                ++mm_cnt;
                tc_fence_after();
                uint32_t wd[32];
                {
                    uint32_t dv[32];
                    tmem_ld32(tB + 64 * hf, dv);
#pragma unroll
                    for (int c2 = 0; c2 < 2; ++c2) {
                        uint32_t wp[16];
#pragma unroll
                        for (int e = 0; e < 16; ++e) wp[e] = pack_bf16(pt[32 * c2 + 2 * e], pt[32 * c2 + 2 * e + 1]);
                        tmem_st16(tB + 64 * hf + 16 * c2, wp);
                    }
                    // dS^T = P^T (dP^T - delta)
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        wd[e] = pack_bf16(pt[2 * e] * (__uint_as_float(dv[2 * e]) - stage[128 + 64 * hf + 2 * e]),
                                          pt[2 * e + 1] * (__uint_as_float(dv[2 * e + 1]) - stage[128 + 64 * hf + 2 * e + 1]));
                }
                {
                    uint32_t dv[32];
                    tmem_ld32(tB + 64 * hf + 32, dv);
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        wd[16 + e] = pack_bf16(
                            pt[32 + 2 * e] * (__uint_as_float(dv[2 * e]) - stage[128 + 64 * hf + 32 + 2 * e]),
                            pt[32 + 2 * e + 1] * (__uint_as_float(dv[2 * e + 1]) - stage[128 + 64 * hf + 32 + 2 * e + 1]));
                }
                // dS^T (bf16) over the half's last 32 columns, read just above
                tmem_st32(tB + 64 * hf + 32, wd);
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar.op_full());
            }
            if (!__all_sync(0xffffffffu, mbar_wait(bar.acc_full(), acc_cnt & 1, st.abort_flag, p.status)))
                goto ew_out;
            ++acc_cnt;
            tc_fence_after();
#pragma unroll
            for (int which = 0; which < 2; ++which) {  // dV, then dK (scaled)
                __nv_bfloat16 *orow = kvalid ? (which ? p.dk : p.dv) + oidx : nullptr;
                const float f = which ? p.scale : 1.f;
#pragma unroll
                for (int cc = hf * (D / 64); cc < (hf + 1) * (D / 64); ++cc) {
                    uint32_t o[32];
                    tmem_ld32((which ? tD : tC) + 32 * cc, o);
                    uint32_t w[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        w[i] = pack_bf16(__uint_as_float(o[2 * i]) * f, __uint_as_float(o[2 * i + 1]) * f);
                    if (orow) {
                        uint4 *dst = reinterpret_cast<uint4 *>(orow + cc * 32);
#pragma unroll
                        for (int v4 = 0; v4 < 4; ++v4)
                            dst[v4] = make_uint4(w[4 * v4], w[4 * v4 + 1], w[4 * v4 + 2], w[4 * v4 + 3]);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar.acc_empty());
        }
    ew_out:;
    }
    teardown<D>(st);
    // Started while the dQ kernel may still run: complete only after it, so
    // that the backward's end on the stream covers dQ as well.
    if (threadIdx.x == 0) grid_dep_wait();
}

}  // namespace bwd
}  // namespace tfa
