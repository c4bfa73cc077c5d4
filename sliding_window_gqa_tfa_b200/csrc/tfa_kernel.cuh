// tfa_kernel.cuh -- persistent, warp-specialised sm_100a kernel for tiled GQA
// prefill attention (online softmax; tcgen05 tensor cores with TMEM
// accumulators; TMA into 128-byte-swizzled shared memory).
//
// What it computes is tiny-llm "Week 2 Day 5: Tiled Dense Prefill Attention"
// (Task 1: per query row an FP32 running max m, sum l and accumulator a merged
// tile by tile as m' = max(m, m_b), l' = e^(m-m') l + e^(m_b-m') l_b,
// a' = e^(m-m') a + e^(m_b-m') a_b, out = a'/l'; Task 2: causality aligned to
// the end of the cached prefix, fully masked rows finite zeros) with the
// sliding window and key mask of brotensor's flash_attention.h.
//
// Work unit ("item"): batch b, query head h and a pair of consecutive 128-row
// query tiles t = 0, 1 (rows [256 qp, 256 qp + 256)).  The two tiles share
// every K/V tile they both reach, and ping-pong on the tensor core: while
// tile 0's softmax runs, the tensor core computes tile 1's products and vice
// versa.  Items are handed out statically to a persistent grid of one CTA per
// SM, longest first (causal items with the most key tiles first), with the
// query heads that share a KV head next to each other so their K/V reads hit L2.
//
// Roles (384 threads, three warpgroups):
//   warps 0-3   softmax + epilogue for query tile 0 (thread = one query row)
//   warps 4-7   softmax + epilogue for query tile 1
//   warp 8      TMA producer (lane 0): Q tiles, then K_j, V_j into a ring of slots
//   warp 9      tensor-core issuer (lane 0)
//   warps 10-11 idle (their registers go to the softmax warpgroups)
// Tensor memory (512 columns, fp32): S_0 [0,128), S_1 [128,256), O_0 and O_1 at
// 256 and 256 + D.  P (bf16, two per column) overwrites S_t's columns [64,128)
// and feeds the P.V product straight from tensor memory.
//
// Per key tile j the issuer runs, for t = 0, 1:  O_t += P_t(j) V_j (after the
// softmax of tile t published P_t(j)), then S_t = Q_t K_{j+1}^T.  tcgen05
// operations from one thread execute in order, so S_t(j+1) never overwrites
// P_t(j) before P_t(j) V_j has read it, and the commit that signals S_t(j+1)
// also covers O_t's update -- the softmax may rescale O_t right after it.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <math_constants.h>

#include "tfa_plan.h"
#include "tfa_ptx.cuh"
#include "tfa_sched.h"

namespace tfa {

// Optional timeline trace of CTA 0 (compile with -DTFA_TRACE; compiled out
// otherwise).  Role r in {0: softmax tile 0, 1: softmax tile 1, 2: MMA issuer,
// 3: TMA producer, 4-7: warps 0-3 of softmax tile 0}; slot = 8 * step + event,
// SM clock.
#ifdef TFA_TRACE
constexpr int kTraceSlots = 2048;
__device__ unsigned long long g_tfa_trace[8][kTraceSlots];
__device__ unsigned long long g_tfa_cta_time[1024][4];  // global-timer ns: start, end, softmax done, packed merge start
#define TFA_TR(role, step, ev)                                                      \
    do {                                                                            \
        const int _i = 8 * (step) + (ev);                                           \
        if (blockIdx.x == 0 && _i < kTraceSlots) g_tfa_trace[role][_i] = clock64(); \
    } while (0)
#else
#define TFA_TR(role, step, ev) \
    do {                       \
    } while (0)
#endif

constexpr int kThreads = 384;
// Registers: the kernel is compiled for 168 per thread at launch (384 x 168 =
// 64512, the most three warps per SM sub-partition can hold).  The producer
// warpgroup then gives back down to kRegsOther and the two softmax
// warpgroups grow to kRegsSoftmax; 2*128*kRegsSoftmax + 128*kRegsOther must not
// exceed 384*kRegsLaunch, or setmaxnreg.inc would wait forever.
constexpr int kRegsLaunch = 168;
constexpr int kRegsSoftmax = 200;
constexpr int kRegsOther = 104;
static_assert(2 * 128 * kRegsSoftmax + 128 * kRegsOther <= kThreads * kRegsLaunch,
              "register split exceeds the launch pool");
// Lazy rescale: keep the stale row maximum until the true one exceeds it by
// more than 2^8 in the exp2 domain (P values then stay <= 256).
constexpr float kRescaleThresholdLog2 = 8.0f;
// The softmax publishes P in two parts: keys [0, kPartKeys) first, so the P.V
// product starts on them while the other keys' exponentials are computed.
// (32 measured 0.5-1.8 % faster than 96 or 64 on the prefill workloads.)
constexpr int kPartKeys = 32;
static_assert(kPartKeys % 32 == 0 && kPartKeys % 16 == 0 && kPartKeys < 128, "P split");

constexpr int kMaxVarlenSeqs = 1024;  // sequences per packed variable-length call

template <int D>
struct Cfg {
    static_assert(D == 64 || D == 128, "head dim");
    static constexpr int kTileBytes = 128 * D * 2;        // 128 rows x D bf16 (Q, K or V tile)
    static constexpr int kColBlocks = D / 64;             // 64-element (128-byte) column blocks
    static constexpr int kColBlockBytes = 128 * 128;      // one 128-row x 128-byte block
    static constexpr int kSlots = (D == 128) ? 4 : 8;     // K/V ring depth
    static constexpr int kQOff = 0;
    static constexpr int kKVOff = 2 * kTileBytes;
    // Key-mask bias: per K/V slot a [128 keys][16] bf16 block whose column 0
    // is 0 (key kept) or -inf (key dropped), and one [128 rows][16] block of
    // "ones" (column 0 = 1); one extra K=16 MMA adds bias[key] to every row of
    // S.  Both blocks are K-major without swizzle (see bias_offset).
    // They sit at the end of the layout: launches without a key mask do not
    // request that shared memory at all (it would shrink the L1 carve-out).
    static constexpr int kBiasBytes = 128 * 16 * 2;
    static constexpr int kBarOff = kKVOff + kSlots * kTileBytes;
    static constexpr int kNumBars = 10 + 2 * kSlots + 1 + 4 + 2 + 1;
    static constexpr int kMiscOff = kBarOff + kNumBars * 8;
    static constexpr int kSmemBytes = kMiscOff + 16 + 1024;  // + slack to align the base to 1 KB
    static constexpr int kBiasOff = ((kMiscOff + 16 + 1023) / 1024) * 1024;
    static constexpr int kOnesOff = kBiasOff + kSlots * kBiasBytes;
    static constexpr int kSmemBytesKeyMask = kOnesOff + kBiasBytes + 1024;
    // Packed variable-length calls: per sequence q_start, q_len, k_start,
    // k_len (validated copies of cu_seqlens), in place of the key-mask blocks
    // (the two never meet).
    static constexpr int kTableOff = kBiasOff;
    // then the sorted sequence order and the group starts of the compact deal
    static constexpr int kOrderOff = kTableOff + 16 * kMaxVarlenSeqs;
    static constexpr int kGroupStartOff = kOrderOff + 4 * kMaxVarlenSeqs;
    static constexpr int kSmemBytesVarlen = kGroupStartOff + 4 * (kMaxVarlenGroups + 1) + 1024;
    static constexpr uint32_t kTmemCols = 512;
    static constexpr uint32_t kTmemS = 0;                 // S_t at kTmemS + 128 t
    static constexpr uint32_t kTmemO = 256;               // O_t at kTmemO + D t
    static constexpr uint32_t kTmemP = 64;                // P_t at S_t + 64
};

struct Params {
    __nv_bfloat16 *o;
    const float *key_mask;
    unsigned *status;
    float *partial;    // split schedule: per (CTA, tile) partial m, l, accumulator
    unsigned *ready;   // split schedule: per (CTA, tile) flag, == the launch's epoch when published
    // logit softcap (kernels instantiated with SC): a raw score x becomes
    // (cap/scale) tanh(u), u = x scale/cap = x * softcap_u, evaluated as
    // softcap_b * (1 - 2 / (2^(x * softcap_a) + 1)) for |u| >= 1/4 and by the
    // odd Taylor series of tanh through u^7 below (no cancellation near 0)
    float softcap_a, softcap_b, softcap_u;
    const float *sinks;  // fp32 [Hq] sink logits, or nullptr
    // rotating cache: K/V hold ring_rows rows and key position j sits in row
    // j mod ring_rows (0: K/V hold all S keys in order)
    int ring_rows;
    // packed variable-length batch (the varlen layout): q/o [total_q, Hq, D],
    // k/v [total_k, Hkv, D], sequence b = rows [cu_q[b], cu_q[b+1]) /
    // [cu_k[b], cu_k[b+1]); shape.L is the longest query (max_seqlen_q)
    int total_q, total_k;
    const int *cu_q, *cu_k;
    // optional per-row log-sum-exp in base 2 of the scaled scores,
    // log2(sum_j 2^(s_j * scale_log2)) (+inf for a row with no allowed key),
    // [B, Hq, L] fp32: what a backward pass needs to rebuild P from S
    float *lse;
    // split schedule: ctl[0] counts finished launches (the epoch of a launch is
    // ctl[0] + 1, read from device memory so a captured graph replays correctly),
    // ctl[1] counts the CTAs of the running launch that have finished
    unsigned *ctl;
    int B, Hq, Hkv, L, S, G;
    int causal, window;
    unsigned flags;
    long long wait_limit;  // SM cycles before a pipeline wait gives up (TFA_WAIT_LIMIT_CYCLES)
    float scale_log2;  // softmax scale * log2(e)
    long long W;       // total key-tile steps (split schedule)
    Shape shape;
    // Short-query (decode) mapping: a query tile holds the rows of pack_heads
    // query heads of one KV group, row m = (head m / L, query row m % L);
    // shape.Hq then counts Hkv * pack_chunks "virtual heads", one per tile.
    int packed, pack_heads, pack_chunks;  // packed: 1 exactly in the PK instantiations
};

// Rows of one packed tile: first real query head, heads present.
struct PackedRows {
    int h0, heads;
};
__device__ __forceinline__ PackedRows packed_rows(const Params &p, int vh) {
    const int g = vh / p.pack_chunks;
    const int hc = vh - g * p.pack_chunks;
    PackedRows pr;
    pr.h0 = g * p.G + hc * p.pack_heads;
    pr.heads = imin(p.pack_heads, p.G - hc * p.pack_heads);
    return pr;
}

// Byte offset of element (row, k) of a [128][16] bf16 K-major block without
// swizzle: core matrices of 8 rows x 16 bytes; the two halves of k 128 bytes
// apart (LBO), consecutive 8-row groups 256 bytes apart (SBO).
__host__ __device__ constexpr uint32_t bias_offset(int row, int k) {
    return (row >> 3) * 256 + (k >> 3) * 128 + (row & 7) * 16 + (k & 7) * 2;
}

// Floats of one partial slot: the accumulator [128][D], then m[128], l[128];
// one slot per (CTA, query tile) (only a CTA's first piece ever publishes).
template <int D>
__host__ __device__ constexpr int partial_slot_floats() { return 128 * D + 256; }
__host__ __device__ constexpr int partial_slot(int cta, int t) { return cta * 2 + t; }

// This launch's epoch (never 0, the flags' initial value).
__device__ __forceinline__ unsigned launch_epoch(const unsigned *ctl) {
    const unsigned e = *reinterpret_cast<const volatile unsigned *>(ctl) + 1u;
    return e == 0u ? 1u : e;
}

// The CTA's dynamic shared memory, 1 KB aligned (the same base the kernel uses).
__device__ __forceinline__ uint8_t *smem_base() {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    return smem_raw + (((raw + 1023u) & ~1023u) - raw);
}

// Where K and V rows live, fixed at compile time so that a dense call carries
// no code for the others: [B*H][rows][D] planes, a rotating cache of ring_rows
// rows per plane, or packed variable-length sequences [total][H][D].
enum Layout : int { kLayoutDense = 0, kLayoutRing = 1, kLayoutVarlen = 2 };

// Start the CTA's piece iterator (with the validated sequence table for a
// packed variable-length call).
template <int D, int LY>
__device__ __forceinline__ void iter_init(SegIter &it, const Params &p) {
    it.init(p.shape, p.W, blockIdx.x);
    if constexpr (LY == kLayoutVarlen) {
        const int *tab = reinterpret_cast<const int *>(smem_base() + Cfg<D>::kTableOff);
        it.seq.q_start = tab;
        it.seq.q_len = tab + kMaxVarlenSeqs;
        it.seq.k_start = tab + 2 * kMaxVarlenSeqs;
        it.seq.k_len = tab + 3 * kMaxVarlenSeqs;
        if (p.shape.n_qp <= kMaxVarlenGroups) {
            it.seq.order = reinterpret_cast<const unsigned *>(smem_base() + Cfg<D>::kOrderOff);
            it.seq.group_start = reinterpret_cast<const int *>(smem_base() + Cfg<D>::kGroupStartOff);
            it.n_items = it.seq.group_start[p.shape.n_qp];
        }
    }
}

struct ItemPlan {
    int b, h, g;
    int q_row0, k_row0;  // varlen: the sequence's first packed query / key row
    int q0[2];
    bool present[2];
    int lo[2], hi[2];
    int jl, jh;
};

// The two query tiles of one piece of work, clipped to the piece's key tiles.
template <bool PK>
__device__ __forceinline__ ItemPlan plan_piece(const Params &p, const Segment &seg) {
    ItemPlan ip;
    ip.b = seg.b;
    ip.h = seg.h;
    // p.packed is tested at run time here and in the producer's Q load (always
    // equal to PK): the compile-time form of these two tests measured ~3 %
    // slower on dense prefill, with identical register and spill counts
    ip.g = (PK || p.packed) ? seg.h / p.pack_chunks : p.shape.hp ? (2 * seg.h) / p.G : seg.h / p.G;
    ip.jl = seg.jb;
    ip.jh = seg.je;
    ip.q_row0 = seg.q_base;
    ip.k_row0 = seg.k_base;
    const ItemSpan sp = seg_span(p.shape, seg);
#pragma unroll
    for (int t = 0; t < 2; ++t) {
        const TileRole tr = tile_role(p.shape, seg, sp, t);
        ip.q0[t] = p.shape.hp ? seg.qp * kBlockQ : seg.qp * 2 * kBlockQ + t * kBlockQ;
        ip.present[t] = tr.active;
        ip.lo[t] = tr.lo;
        ip.hi[t] = tr.active ? tr.hi : -1;
    }
    return ip;
}

struct Bars {
    uint32_t base;
    int slots;
    __device__ __forceinline__ uint32_t q_full(int t) const { return base + 8 * (0 + t); }
    __device__ __forceinline__ uint32_t q_empty(int t) const { return base + 8 * (2 + t); }
    __device__ __forceinline__ uint32_t s_full(int t) const { return base + 8 * (4 + t); }
    __device__ __forceinline__ uint32_t p_full(int t) const { return base + 8 * (6 + t); }
    __device__ __forceinline__ uint32_t o_full(int t) const { return base + 8 * (8 + t); }
    __device__ __forceinline__ uint32_t kv_full(int s) const { return base + 8 * (10 + s); }
    __device__ __forceinline__ uint32_t kv_empty(int s) const { return base + 8 * (10 + slots + s); }
    __device__ __forceinline__ uint32_t done() const { return base + 8 * (10 + 2 * slots); }
    // split schedule: the four warps of tile t stored their partial / the
    // finalizer thread saw every contributor's flag
    __device__ __forceinline__ uint32_t pub(int t) const { return base + 8 * (11 + 2 * slots + t); }
    __device__ __forceinline__ uint32_t fin(int t) const { return base + 8 * (13 + 2 * slots + t); }
    // P_t's first kPartKeys key columns are in tensor memory (the P.V product
    // may start on them while the softmax finishes the rest)
    __device__ __forceinline__ uint32_t p_part(int t) const { return base + 8 * (15 + 2 * slots + t); }
    // packed tiles: one step of a finalizer's merge, the four warps of tile 0 arriving
    __device__ __forceinline__ uint32_t merge_step() const { return base + 8 * (17 + 2 * slots); }
};

// ------------------------------------------------------------------ producer
template <int D, bool KM, int LY, bool PK>
__device__ void load_role(const Params &p, const CUtensorMap *tm_q, const CUtensorMap *tm_k,
                          const CUtensorMap *tm_v, uint32_t sbase, uint8_t *gbase, const Bars &bar,
                          volatile int *abort_flag) {
    // With a key mask the whole warp runs this loop (lane 0 issues the copies
    // and arms the barriers, all lanes write each K tile's bias); without one
    // only lane 0 does.
    using C = Cfg<D>;
    const int lane = threadIdx.x & 31;
    constexpr bool has_km = KM;
    constexpr unsigned lanes = KM ? 0xffffffffu : 1u;
    uint32_t kv_prod = 0;
    uint32_t q_use[2] = {0, 0};
    SegIter it;
    iter_init<D, LY>(it, p);
    // K/V tiles are read again by the other CTAs of their KV group (and the
    // other query tiles); Q tiles are read once.  Marking them evict-last /
    // evict-first keeps K/V in L2 while Q and O stream through it.
    const uint64_t pol_kv = make_policy_evict_last(), pol_q = make_policy_evict_first();
    Segment seg;
    while (it.next(p.shape, seg)) {
        const ItemPlan ip = plan_piece<PK>(p, seg);
#pragma unroll
        for (int t = 0; t < 2; ++t) {
            if (!ip.present[t]) continue;
            if (q_use[t] > 0 &&
                !__all_sync(lanes, mbar_wait(bar.q_empty(t), (q_use[t] - 1) & 1, abort_flag, p.status, p.wait_limit)))
                goto out;
            if (lane == 0) {
                if (PK || p.packed) {  // box {64, L, pack_heads}: rows (head, query row) in order
                    const PackedRows pr = packed_rows(p, ip.h);
                    mbar_arrive_expect_tx(bar.q_full(t), C::kColBlocks * 128 * p.L * p.pack_heads);
                    for (int cb = 0; cb < C::kColBlocks; ++cb)
                        tma_load_3d_hint(sbase + C::kQOff + t * C::kTileBytes + cb * C::kColBlockBytes,
                                         tm_q, bar.q_full(t), cb * 64, 0, ip.b * p.Hq + pr.h0, pol_q);
                } else {  // dense: plane b*Hq + h (head pairs: 2h + t); varlen: packed rows, plane h
                    mbar_arrive_expect_tx(bar.q_full(t), C::kTileBytes);
                    const int head = p.shape.hp ? 2 * ip.h + t : ip.h;
                    const int plane = LY == kLayoutVarlen ? head : ip.b * p.Hq + head;
                    for (int cb = 0; cb < C::kColBlocks; ++cb)
                        tma_load_3d_hint(sbase + C::kQOff + t * C::kTileBytes + cb * C::kColBlockBytes,
                                         tm_q, bar.q_full(t), cb * 64, ip.q_row0 + ip.q0[t], plane, pol_q);
                }
            }
            ++q_use[t];
        }
        for (int j = ip.jl; j <= ip.jh; ++j) {
            for (int which = 0; which < 2; ++which) {  // K_j then V_j
                const uint32_t s = kv_prod % C::kSlots;
                const uint32_t round = kv_prod / C::kSlots;
                if (round > 0 &&
                    !__all_sync(lanes, mbar_wait(bar.kv_empty(s), (round - 1) & 1, abort_flag, p.status, p.wait_limit)))
                    goto out;
                if (which == 0 && has_km) {
                    // bias column of this K tile: 0 for kept keys, -inf otherwise
                    const float *km_row = p.key_mask + static_cast<size_t>(ip.b) * p.S;
                    uint8_t *blk = gbase + C::kBiasOff + s * C::kBiasBytes;
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int n = 32 * i + lane;
                        const int key = j * kBlockK + n;
                        const bool keep = key < p.S && __ldg(km_row + key) > 0.5f;
                        *reinterpret_cast<uint16_t *>(blk + bias_offset(n, 0)) = keep ? 0x0000u : 0xFF80u;
                    }
                    fence_proxy_async_smem();  // the tensor core reads it through the async proxy
                    __syncwarp();
                }
                if (lane == 0) {
                    mbar_arrive_expect_tx(bar.kv_full(s), C::kTileBytes);
                    const uint32_t dst = sbase + C::kKVOff + s * C::kTileBytes;
                    if constexpr (LY == kLayoutRing) {
                        // rotating cache: two 64-row boxes, each contiguous in
                        // the ring (ring_rows is a multiple of 64)
                        for (int hf = 0; hf < 2; ++hf) {
                            const int row = (j * kBlockK + 64 * hf) % p.ring_rows;
                            for (int cb = 0; cb < C::kColBlocks; ++cb)
                                tma_load_3d_hint(dst + cb * C::kColBlockBytes + hf * 64 * 128, which ? tm_v : tm_k,
                                                 bar.kv_full(s), cb * 64, row, ip.b * p.Hkv + ip.g, pol_kv);
                        }
                    } else {
                        const int plane = LY == kLayoutVarlen ? ip.g : ip.b * p.Hkv + ip.g;
                        for (int cb = 0; cb < C::kColBlocks; ++cb)
                            tma_load_3d_hint(dst + cb * C::kColBlockBytes, which ? tm_v : tm_k, bar.kv_full(s),
                                             cb * 64, ip.k_row0 + j * kBlockK, plane, pol_kv);
                    }
                }
                ++kv_prod;
            }
        }
    }
out:
    if (lane != 0) return;
    // Every copy lane 0 started must land before the CTA may exit.
    for (uint32_t s = 0; s < (uint32_t)C::kSlots; ++s) {
        if (kv_prod > s) {
            const uint32_t armed = (kv_prod - s - 1) / C::kSlots + 1;
            mbar_drain(bar.kv_full(s), (armed - 1) & 1);
        }
    }
    for (int t = 0; t < 2; ++t)
        if (q_use[t] > 0) mbar_drain(bar.q_full(t), (q_use[t] - 1) & 1);
}

// ------------------------------------------------------------ tensor cores
template <int D, bool KM, int LY, bool PK>
__device__ void mma_role(const Params &p, uint32_t sbase, uint32_t tmem, const Bars &bar,
                         volatile int *abort_flag) {
    using C = Cfg<D>;
    constexpr uint32_t kIdescQK = idesc_bf16_f32(128, kBlockK, 0);  // S = Q K^T, both K-major
    constexpr uint32_t kIdescPV = idesc_bf16_f32(128, D, 1);        // O += P V, V MN-major
    const uint32_t q_smem = sbase + C::kQOff;
    const uint32_t kv_smem = sbase + C::kKVOff;
    constexpr bool has_km = KM;

    // Descriptors are built once: the start-address field holds address >> 4
    // in its low 14 bits, so moving an operand by `off` bytes (shared memory
    // stays below 256 KB) adds off >> 4 to the 64-bit descriptor.
    // S_t = Q_t K^T: A = Q tile, B = K tile, both [128 rows][D] K-major with
    // 128-byte swizzle; a K-step of 16 elements advances 32 bytes inside a
    // 128-byte row and moves to the next column block every 4 steps.
    const uint64_t dq0 = smem_desc_sw128(q_smem, 16, 1024);
    const uint64_t dkv0 = smem_desc_sw128(kv_smem, 16, 1024);
    // O_t += P_t V: A = P_t in tensor memory (8 columns per 16 keys), B = V tile
    // read MN-major (D contiguous): 8 key rows per 1 KB swizzle atom (SBO), the
    // next 64 head-dim columns one column block further (LBO).
    const uint64_t dv0 = smem_desc_sw128(kv_smem, C::kColBlockBytes, 1024);
    uint64_t d_ones = 0, d_bias0 = 0;
    if constexpr (KM) {
        d_ones = smem_desc_noswizzle(sbase + C::kOnesOff, 128, 256);
        d_bias0 = smem_desc_noswizzle(sbase + C::kBiasOff, 128, 256);
    }
    constexpr uint32_t kTileStep = C::kTileBytes >> 4;
    auto issue_qk = [&](int t, uint32_t slot) {
        const uint64_t dq = dq0 + t * kTileStep;
        const uint64_t dk = dkv0 + slot * kTileStep;
        const uint32_t d_tmem = tmem + C::kTmemS + t * 128;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = ((kk >> 2) * C::kColBlockBytes + (kk & 3) * 32) >> 4;
            umma_ss(d_tmem, dq + off, dk + off, kIdescQK, kk > 0 ? 1u : 0u);
        }
        if constexpr (has_km)  // S += ones * bias^T: the key mask as a per-column 0 / -inf
            umma_ss(d_tmem, d_ones, d_bias0 + slot * (C::kBiasBytes >> 4), kIdescQK, 1u);
    };
    auto issue_pv = [&](int t, uint32_t slot, bool accumulate, int kk_begin, int kk_end) {
        const uint64_t dv = dv0 + slot * kTileStep;
        const uint32_t d_tmem = tmem + C::kTmemO + t * D;
        const uint32_t a_tmem = tmem + C::kTmemS + t * 128 + C::kTmemP;
        for (int kk = kk_begin; kk < kk_end; ++kk)
            umma_ts(d_tmem, a_tmem + kk * 8, dv + kk * ((16 * 128) >> 4), kIdescPV,
                    (accumulate || kk > 0) ? 1u : 0u);
    };

    uint32_t kv_cons = 0;
    uint32_t q_use[2] = {0, 0};
    uint32_t p_cnt[2] = {0, 0};
    int trace_step = 0;
    (void)trace_step;
    SegIter it;
    iter_init<D, LY>(it, p);
    Segment seg;
    if constexpr (PK) {
        // Short-query tiles: one query tile (tile 0) whose score tiles
        // alternate between the two S buffers, so S_{j+1} = Q K_{j+1}^T is
        // computed while the softmax works on S_j.  P.V products then finish
        // after the next score tile's: each but the piece's last commits to
        // o_full(1) (tile 1 never exists here), which the softmax waits on
        // before it may rescale O.
        auto qk_to = [&](int buf, uint32_t slot) {
            const uint64_t dk = dkv0 + slot * kTileStep;
            const uint32_t d_tmem = tmem + C::kTmemS + buf * 128;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t off = ((kk >> 2) * C::kColBlockBytes + (kk & 3) * 32) >> 4;
                umma_ss(d_tmem, dq0 + off, dk + off, kIdescQK, kk > 0 ? 1u : 0u);
            }
            if constexpr (has_km) umma_ss(d_tmem, d_ones, d_bias0 + slot * (C::kBiasBytes >> 4), kIdescQK, 1u);
        };
        auto pv_from = [&](int buf, uint32_t slot, bool accumulate, int kk_begin, int kk_end) {
            const uint64_t dv = dv0 + slot * kTileStep;
            const uint32_t a_tmem = tmem + C::kTmemS + buf * 128 + C::kTmemP;
            for (int kk = kk_begin; kk < kk_end; ++kk)
                umma_ts(tmem + C::kTmemO, a_tmem + kk * 8, dv + kk * ((16 * 128) >> 4), kIdescPV,
                        (accumulate || kk > 0) ? 1u : 0u);
        };
        while (it.next(p.shape, seg)) {
            const ItemPlan ip = plan_piece<PK>(p, seg);
            if (ip.jl > ip.jh) continue;  // no key tile: nothing was loaded
            if (!mbar_wait(bar.q_full(0), q_use[0] & 1, abort_flag, p.status, p.wait_limit)) goto out;
            ++q_use[0];
            {
                const uint32_t s = kv_cons % C::kSlots;
                if (!mbar_wait(bar.kv_full(s), (kv_cons / C::kSlots) & 1, abort_flag, p.status, p.wait_limit)) goto out;
                ++kv_cons;
                tc_fence_after();
                qk_to(0, s);
                umma_commit(bar.s_full(0));
                if (ip.jl == ip.jh) umma_commit(bar.q_empty(0));
                umma_commit(bar.kv_empty(s));
            }
            for (int j = ip.jl; j <= ip.jh; ++j) {
                TFA_TR(2, trace_step, 0);
                const int buf = (j - ip.jl) & 1;
                const uint32_t sv = kv_cons % C::kSlots;
                if (!mbar_wait(bar.kv_full(sv), (kv_cons / C::kSlots) & 1, abort_flag, p.status, p.wait_limit)) goto out;
                ++kv_cons;
                if (j < ip.jh) {
                    const uint32_t sk = kv_cons % C::kSlots;
                    if (!mbar_wait(bar.kv_full(sk), (kv_cons / C::kSlots) & 1, abort_flag, p.status, p.wait_limit)) goto out;
                    ++kv_cons;
                    tc_fence_after();
                    TFA_TR(2, trace_step, 1);
                    qk_to(buf ^ 1, sk);
                    umma_commit(bar.s_full(buf ^ 1));
                    if (j + 1 == ip.jh) umma_commit(bar.q_empty(0));
                    umma_commit(bar.kv_empty(sk));
                }
                if (!mbar_wait(bar.p_part(0), p_cnt[0] & 1, abort_flag, p.status, p.wait_limit)) goto out;
                TFA_TR(2, trace_step, 2);
                tc_fence_after();
                pv_from(buf, sv, j > ip.jl, 0, kPartKeys / 16);
                if (!mbar_wait(bar.p_full(0), p_cnt[0] & 1, abort_flag, p.status, p.wait_limit)) goto out;
                TFA_TR(2, trace_step, 3);
                ++p_cnt[0];
                tc_fence_after();
                pv_from(buf, sv, true, kPartKeys / 16, kBlockK / 16);
                ++trace_step;
                umma_commit(j == ip.jh ? bar.o_full(0) : bar.o_full(1));
                umma_commit(bar.kv_empty(sv));
            }
        }
    } else {
        while (it.next(p.shape, seg)) {
            const ItemPlan ip = plan_piece<PK>(p, seg);
#pragma unroll
            for (int t = 0; t < 2; ++t) {
                if (!ip.present[t]) continue;
                if (!mbar_wait(bar.q_full(t), q_use[t] & 1, abort_flag, p.status, p.wait_limit)) goto out;
                ++q_use[t];
            }
            {
                const uint32_t s = kv_cons % C::kSlots;
                if (!mbar_wait(bar.kv_full(s), (kv_cons / C::kSlots) & 1, abort_flag, p.status, p.wait_limit)) goto out;
                ++kv_cons;
                tc_fence_after();
#pragma unroll
                for (int t = 0; t < 2; ++t) {
                    if (ip.present[t] && ip.lo[t] <= ip.jl) {
                        issue_qk(t, s);
                        umma_commit(bar.s_full(t));
                        if (ip.hi[t] == ip.jl) umma_commit(bar.q_empty(t));
                    }
                }
                umma_commit(bar.kv_empty(s));
            }
            bool acc[2] = {false, false};
            for (int j = ip.jl; j <= ip.jh; ++j) {
                TFA_TR(2, trace_step, 0);
                const uint32_t sv = kv_cons % C::kSlots;
                if (!mbar_wait(bar.kv_full(sv), (kv_cons / C::kSlots) & 1, abort_flag, p.status, p.wait_limit)) goto out;
                ++kv_cons;
                const bool next = j < ip.jh;
                uint32_t sk = 0;
                if (next) {
                    sk = kv_cons % C::kSlots;
                    if (!mbar_wait(bar.kv_full(sk), (kv_cons / C::kSlots) & 1, abort_flag, p.status, p.wait_limit))
                        goto out;
                    ++kv_cons;
                }
                TFA_TR(2, trace_step, 1);
                tc_fence_after();
#pragma unroll
                for (int t = 0; t < 2; ++t) {
                    if (!ip.present[t]) continue;
                    if (ip.lo[t] <= j && j <= ip.hi[t]) {
                        // first part of P_t, then the rest (the tensor core works on
                        // the first part meanwhile)
                        if (!mbar_wait(bar.p_part(t), p_cnt[t] & 1, abort_flag, p.status, p.wait_limit)) goto out;
                        TFA_TR(2, trace_step, 2 + 2 * t);
                        tc_fence_after();
                        issue_pv(t, sv, acc[t], 0, kPartKeys / 16);
                        if (!mbar_wait(bar.p_full(t), p_cnt[t] & 1, abort_flag, p.status, p.wait_limit)) goto out;
                        ++p_cnt[t];
                        tc_fence_after();
                        issue_pv(t, sv, true, kPartKeys / 16, kBlockK / 16);
                        acc[t] = true;
                        if (j == ip.hi[t]) umma_commit(bar.o_full(t));
                    }
                    if (next && ip.lo[t] <= j + 1 && j + 1 <= ip.hi[t]) {
                        issue_qk(t, sk);
                        umma_commit(bar.s_full(t));
                        if (j + 1 == ip.hi[t]) umma_commit(bar.q_empty(t));
                    }
                    TFA_TR(2, trace_step, 3 + 2 * t);
                }
                ++trace_step;
                umma_commit(bar.kv_empty(sv));
                if (next) umma_commit(bar.kv_empty(sk));
            }
        }
    }
out:
    // Nothing may leave tensor memory in flight when the CTA frees it.
    umma_commit(bar.done());
    mbar_drain(bar.done(), 0);
}

// ---------------------------------------------------- softmax and epilogue
constexpr float kLog2e = 1.4426950408889634f;

// The row sum with the attention sink's term (a logit with no value row) for
// output head `head`, against reference maximum m (raw-score units).
__device__ __forceinline__ float add_sink(const Params &p, float l, float m, float c, int head) {
    if (p.sinks == nullptr || m == -CUDART_INF_F) return l;  // an empty row stays 0
    return l + ex2(fmaf(__ldg(p.sinks + head), kLog2e, -m * c));
}

// Epilogue / score variants of the kernel, fixed at compile time so that a
// plain call carries no code for the others: a softcap on the scores, or the
// per-row log-sum-exp written beside the output (for a backward pass).
enum ScoreMode : int { kModePlain = 0, kModeSoftcap = 1, kModeLse = 2 };

// Finalizer of a cut packed (short-query) tile, run by the 128 threads of
// tile 0's warpgroup once each has stored its row of the finalizer's own
// partial in this CTA's second slot (the first may still hold the partial
// this CTA published for an earlier tile): the merge of all the tile's
// partials (tiny-llm Week 2 Day 5, Task 1: m* = max m_k,
// l* = sum 2^(m_k - m*) l_k, a* = sum 2^(m_k - m*) a_k, O = a* / l*),
// written straight to the output.  A packed tile has few live rows but one
// partial per CTA of its key range, so the threads split the flag waits and
// the (row, 4-column) elements between them instead of one thread walking
// every partial of its row; each thread merges its elements' statistics
// itself, batch by batch with the same equations (one L2 round trip per
// batch of partials, no step between statistics and elements).  The threads
// meet once, after the flag waits, at an mbarrier with bounded waits (never a
// named barrier: a warp that gave up early must not leave the others
// waiting).  `steps` counts the merge_step phases this thread has passed.
// Returns false on an abort.
template <int D, int MODE>
__device__ __forceinline__ bool merge_packed(const Params &p, const Segment &seg, const ItemSpan &sp,
                                          int n_valid, unsigned epoch, volatile int *abort_flag,
                                          const Bars &bar, uint32_t &steps) {
    constexpr int kN = 128;  // merging threads
    const int r = threadIdx.x;
    const int lane = threadIdx.x & 31;
    const float c = p.scale_log2;
    const int c_last = last_contributor(p.W, gridDim.x, blockIdx.x, seg, sp, 0);
#ifdef TFA_TRACE
    if (r == 0 && blockIdx.x < 1024) g_tfa_cta_time[blockIdx.x][3] = globaltimer_ns();
#endif
    for (int k = blockIdx.x + 1 + r; k <= c_last; k += kN)
        if (!flag_wait(p.ready + partial_slot(k, 0), epoch, abort_flag, p.status, p.wait_limit)) break;
    // every warp arrives, then every lane waits (bounded): the slot writes of
    // tile 0's warps and the flags seen here are ordered before every read
    // below; all threads leave together on an abort, a timed-out wait raising it
    __syncwarp();
    if (lane == 0) mbar_arrive(bar.merge_step());
    const bool met = __all_sync(0xffffffffu, mbar_wait(bar.merge_step(), steps & 1, abort_flag, p.status,
                                                       p.wait_limit));
    ++steps;
    if (!met || *abort_flag) return false;
    auto slot_of = [&](int k) {
        return p.partial +
               static_cast<size_t>(partial_slot(k, k == static_cast<int>(blockIdx.x) ? 1 : 0)) * partial_slot_floats<D>();
    };
    const PackedRows pr = packed_rows(p, seg.h);
    constexpr int kC4 = D / 4;  // float4 columns per row
    const int n4 = n_valid * kC4;
    for (int e0 = r; e0 < n4; e0 += 2 * kN) {  // two elements per thread per pass
        const int e1 = e0 + kN;
        const bool has1 = e1 < n4;
        const int row0 = e0 / kC4, row1 = has1 ? e1 / kC4 : row0;
        const int c40 = e0 - row0 * kC4, c41 = has1 ? e1 - row1 * kC4 : c40;
        float m0 = -CUDART_INF_F, m1 = -CUDART_INF_F, l0 = 0.f, l1 = 0.f;
        float4 a0 = make_float4(0.f, 0.f, 0.f, 0.f), a1 = a0;
        // batches of partials, loads predicated (not a remainder loop) so that
        // a batch's loads are all in flight together however few there are
        constexpr int kBatch = 8;
        for (int k0 = blockIdx.x; k0 <= c_last; k0 += kBatch) {
            float mk0[kBatch], mk1[kBatch], lk0[kBatch], lk1[kBatch];
            float4 v0[kBatch], v1[kBatch];
#pragma unroll
            for (int u = 0; u < kBatch; ++u) {
                const bool in = k0 + u <= c_last;
                const float *sl = slot_of(in ? k0 + u : k0);
                mk0[u] = in ? __ldcg(sl + 128 * D + row0) : -CUDART_INF_F;
                mk1[u] = in ? __ldcg(sl + 128 * D + row1) : -CUDART_INF_F;
                lk0[u] = in ? __ldcg(sl + 128 * D + 128 + row0) : 0.f;
                lk1[u] = in ? __ldcg(sl + 128 * D + 128 + row1) : 0.f;
                v0[u] = __ldcg(reinterpret_cast<const float4 *>(sl + row0 * D) + c40);
                v1[u] = __ldcg(reinterpret_cast<const float4 *>(sl + row1 * D) + c41);
            }
            float mb0 = m0, mb1 = m1;
#pragma unroll
            for (int u = 0; u < kBatch; ++u) mb0 = fmaxf(mb0, mk0[u]), mb1 = fmaxf(mb1, mk1[u]);
            // an empty row (every m -inf) keeps l = 0 and a = 0
            const float nb0 = (mb0 == -CUDART_INF_F) ? 0.f : mb0 * c, nb1 = (mb1 == -CUDART_INF_F) ? 0.f : mb1 * c;
            const float g0 = (m0 == -CUDART_INF_F) ? 0.f : ex2(fmaf(m0, c, -nb0));
            const float g1 = (m1 == -CUDART_INF_F) ? 0.f : ex2(fmaf(m1, c, -nb1));
            l0 *= g0, l1 *= g1;
            a0.x *= g0, a0.y *= g0, a0.z *= g0, a0.w *= g0;
            a1.x *= g1, a1.y *= g1, a1.z *= g1, a1.w *= g1;
#pragma unroll
            for (int u = 0; u < kBatch; ++u) {
                const float f0 = (mk0[u] == -CUDART_INF_F) ? 0.f : ex2(fmaf(mk0[u], c, -nb0));
                const float f1 = (mk1[u] == -CUDART_INF_F) ? 0.f : ex2(fmaf(mk1[u], c, -nb1));
                l0 = fmaf(f0, lk0[u], l0), l1 = fmaf(f1, lk1[u], l1);
                a0.x = fmaf(f0, v0[u].x, a0.x), a0.y = fmaf(f0, v0[u].y, a0.y);
                a0.z = fmaf(f0, v0[u].z, a0.z), a0.w = fmaf(f0, v0[u].w, a0.w);
                a1.x = fmaf(f1, v1[u].x, a1.x), a1.y = fmaf(f1, v1[u].y, a1.y);
                a1.z = fmaf(f1, v1[u].z, a1.z), a1.w = fmaf(f1, v1[u].w, a1.w);
            }
            m0 = mb0, m1 = mb1;
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            if (u == 1 && !has1) break;
            const int rr = u ? row1 : row0, c4 = u ? c41 : c40;
            const float4 a = u ? a1 : a0;
            const int head = pr.h0 + rr / p.L, row = rr % p.L;
            const float m = u ? m1 : m0;
            const float l = add_sink(p, u ? l1 : l0, m, c, head);
            if (MODE == kModeLse && c4 == 0)
                p.lse[static_cast<size_t>(seg.b * p.Hq + head) * p.L + row] =
                    l > 0.f ? fmaf(m, c, __log2f(l)) : CUDART_INF_F;
            const float inv = l > 0.f ? 1.f / l : 0.f;
            __nv_bfloat16 *orow = p.o + (static_cast<size_t>(seg.b * p.Hq + head) * p.L + row) * D;
            *reinterpret_cast<uint2 *>(orow + 4 * c4) = make_uint2(pack_bf16(a.x * inv, a.y * inv),
                                                                  pack_bf16(a.z * inv, a.w * inv));
        }
    }
    return true;
}

template <int D, bool KM, int MODE, int LY, bool PK>
__device__ __forceinline__ void softmax_role(const Params &p, const int t, uint32_t tmem,
                                          const Bars &bar, volatile int *abort_flag) {
    using C = Cfg<D>;
    constexpr bool SC = MODE == kModeSoftcap;
    const int r = threadIdx.x - t * 128;  // row inside the query tile
    const uint32_t lane_base = (static_cast<uint32_t>((threadIdx.x >> 5) & 3) * 32u) << 16;
    const uint32_t tS = tmem + C::kTmemS + t * 128 + lane_base;
    const uint32_t tP = tS + C::kTmemP;
    const uint32_t tO = tmem + C::kTmemO + t * D + lane_base;
    const float c = p.scale_log2;
    const int lane = threadIdx.x & 31;
    uint32_t s_cnt = 0, o_cnt = 0, pub_cnt = 0, fin_cnt = 0;
    uint32_t s_cnt0 = 0, s_cnt1 = 0, pv_cnt = 0;  // short-query tiles: per S buffer, P.V done
    uint32_t merge_steps = 0;                      // short-query tiles: merge steps passed
    const unsigned epoch = p.ctl ? launch_epoch(p.ctl) : 0u;
    int trace_step = 0;
    (void)trace_step;

    SegIter it;
    iter_init<D, LY>(it, p);
    Segment seg;
    while (it.next(p.shape, seg)) {
        const ItemSpan sp = seg_span(p.shape, seg);
        const TileRole ip = tile_role(p.shape, seg, sp, t);
        if (!ip.active) continue;
        // query row of this thread (its head too, for a packed tile)
        int row = p.shape.hp ? seg.qp * kBlockQ + r : seg.qp * 2 * kBlockQ + t * kBlockQ + r;
        int out_head = p.shape.hp ? 2 * seg.h + t : seg.h;
        bool row_valid = row < seg.L;
        const int q_tile0 = row - r;  // first row of the tile, for the tile-level mask test
        if constexpr (PK) {
            const PackedRows pr = packed_rows(p, seg.h);
            row = r % p.L;
            out_head = pr.h0 + r / p.L;
            row_valid = r < pr.heads * p.L;
        }
        const int pos = (seg.S - seg.L) + row;  // absolute position of this query row
        const int hi_abs = p.causal ? imin(pos, seg.S - 1) : seg.S - 1;
        const int lo_abs = (p.causal && p.window > 0) ? pos - p.window + 1 : 0;
        float m_ref = -CUDART_INF_F;  // row maximum the exponentials are taken against
        float l = 0.f;
        bool first = true;

        for (int j = ip.lo; j <= ip.hi; ++j) {
            if (r == 0) TFA_TR(t, trace_step, 0);
            // short-query tiles alternate between the two S buffers
            uint32_t tSj = tS, tPj = tP, sph;
            int sb = t;
            if constexpr (PK) {
                sb = (j - ip.lo) & 1;
                tSj = tS + sb * 128;
                tPj = tP + sb * 128;
                sph = (sb ? s_cnt1++ : s_cnt0++) & 1;
            } else {
                sph = s_cnt++ & 1;
            }
            // all lanes leave together: the tcgen05 loads below are warp-collective
            if (!__all_sync(0xffffffffu, mbar_wait(bar.s_full(sb), sph, abort_flag, p.status, p.wait_limit)))
                return;
            if (r == 0) TFA_TR(t, trace_step, 1);
            tc_fence_after();
            uint32_t s[128];
            tmem_ld128(tSj, s);
            if (r == 0) TFA_TR(t, trace_step, 2);
            if constexpr (SC) {
                // Gemma-2 logit softcap (brotensor flash_attention.h): the scaled
                // score t becomes cap * tanh(t / cap), before masks and softmax;
                // kept in raw-score units so the exponent below is unchanged.
                const float a = p.softcap_a, b = p.softcap_b, us = p.softcap_u, nb2 = -2.f * p.softcap_b;
#pragma unroll
                for (int i = 0; i < 128; ++i) {
                    const float x = __uint_as_float(s[i]);
                    const float far = fmaf(nb2, rcp_approx(ex2(x * a) + 1.f), b);
                    const float u = x * us, u2 = u * u;
                    // tanh u = u - u^3/3 + 2u^5/15 - 17u^7/315 + O(u^9)
                    const float series = u * fmaf(u2, fmaf(u2, fmaf(u2, -17.f / 315.f, 2.f / 15.f), -1.f / 3.f), 1.f);
                    float y = fabsf(u) < 0.25f ? series * b : far;
                    if (KM) y = (x == -CUDART_INF_F) ? x : y;  // a key-masked score stays -inf
                    s[i] = __float_as_uint(y);
                }
            }
            if (t == 0 && lane == 0) TFA_TR(4 + (r >> 5), trace_step, 0);

            if (key_tile_needs_mask(seg.L, seg.S, p.causal, p.window, 0, q_tile0, j, p.flags)) {
                const int k0 = j * kBlockK;
                const int lo_c = lo_abs - k0;
                const int hi_c = hi_abs - k0;
#pragma unroll
                for (int cidx = 0; cidx < 128; ++cidx) {
                    // causal / window / key-tail predicate; the key mask arrived
                    // through the bias MMA already
                    const bool keep = cidx >= lo_c && cidx <= hi_c;
                    if (!keep) s[cidx] = 0xff800000u;  // -inf
                }
            }

            // row maximum: three-input max in four independent chains
#define TFA_F(i) __uint_as_float(s[i])
            float mx[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) mx[k] = fmaxf(TFA_F(k), TFA_F(k + 8));
#pragma unroll
            for (int i = 16; i < 128; i += 16) {
#pragma unroll
                for (int k = 0; k < 8; ++k) mx[k] = fmax3(mx[k], TFA_F(i + k), TFA_F(i + k + 8));
            }
            const float m_new = fmax3(m_ref, fmax3(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], mx[5]),
                                                   fmaxf(mx[6], mx[7])), -CUDART_INF_F);
            if (t == 0 && lane == 0) TFA_TR(4 + (r >> 5), trace_step, 1);

            // Decide the lazy rescale first; O_t itself is rescaled after P is
            // stored, once the S registers are dead.
            float alpha = 1.f;
            bool rescale = false;
            if (first) {
                m_ref = m_new;  // the first P.V overwrites O, nothing to rescale
                first = false;
            } else {
                // (m_new - m_ref) is NaN when both are -inf (row still empty: keep),
                // +inf when the row sees its first key (rescale by 0).
                const bool need = (m_new - m_ref) * c > kRescaleThresholdLog2;
                rescale = __any_sync(0xffffffffu, need);
                if (need) {
                    alpha = (m_ref == -CUDART_INF_F) ? 0.f : ex2((m_ref - m_new) * c);
                    m_ref = m_new;
                }
            }

            // O_t must be rescaled before any of P_t is published: the P.V
            // product may start as soon as the first part is.
            if constexpr (PK) {
                // the previous tile's P.V product may still be accumulating
                if (j > ip.lo) {
                    if (!__all_sync(0xffffffffu, mbar_wait(bar.o_full(1), pv_cnt & 1, abort_flag, p.status, p.wait_limit)))
                        return;
                    ++pv_cnt;
                    tc_fence_after();
                }
            }
            if (rescale) {  // rare; 8 columns at a time while the scores are live
                for (int cc = 0; cc < D / 8; ++cc) {
                    uint32_t o[8];
                    tmem_ld8(tO + cc * 8, o);
#pragma unroll
                    for (int i = 0; i < 8; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
                    tmem_st8(tO + cc * 8, o);
                }
            }

            const float mc = (m_ref == -CUDART_INF_F) ? 0.f : m_ref * c;
            const float2 c2 = make_float2(c, c), nmc2 = make_float2(-mc, -mc);
            float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
            uint32_t pk[64];
#define TFA_EXP_PAIR(i)                                                                    \
    do {                                                                                   \
        const float2 x = fma2(make_float2(TFA_F(2 * (i)), TFA_F(2 * (i) + 1)), c2, nmc2);  \
        float2 e;                                                                          \
        e.x = ex2(x.x); /* MUFU */                                                         \
        e.y = ex2(x.y);                                                                    \
        if ((i) & 1)                                                                       \
            acc1 = add2(acc1, e);                                                          \
        else                                                                               \
            acc0 = add2(acc0, e);                                                          \
        pk[i] = pack_bf16(e.x, e.y);                                                       \
    } while (0)
            // keys [0, kPartKeys): publish, then the rest
#pragma unroll
            for (int i = 0; i < kPartKeys / 2; ++i) TFA_EXP_PAIR(i);
            if (t == 0 && lane == 0) TFA_TR(4 + (r >> 5), trace_step, 3);
#pragma unroll
            for (int c32 = 0; c32 < kPartKeys / 64; ++c32) tmem_st32(tPj + 32 * c32, pk + 32 * c32);
            if ((kPartKeys / 2) % 32) tmem_st16(tPj + (kPartKeys / 64) * 32, pk + (kPartKeys / 64) * 32);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar.p_part(t));
            if (t == 0 && lane == 0) TFA_TR(4 + (r >> 5), trace_step, 4);
#pragma unroll
            for (int i = kPartKeys / 2; i < 64; ++i) TFA_EXP_PAIR(i);
            if (t == 0 && lane == 0) TFA_TR(4 + (r >> 5), trace_step, 5);
#undef TFA_EXP_PAIR
#undef TFA_F
            const float2 acc = add2(acc0, acc1);
            l = l * alpha + (acc.x + acc.y);
#pragma unroll
            for (int c16 = kPartKeys / 32; c16 < 4; ++c16) tmem_st16(tPj + 16 * c16, pk + 16 * c16);
            if (r == 0) TFA_TR(t, trace_step, 3);
            if (t == 0 && lane == 0) TFA_TR(4 + (r >> 5), trace_step, 2);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar.p_full(t));  // one arrival per warp
            if (r == 0) TFA_TR(t, trace_step, 4);
            ++trace_step;
        }

        if (!__all_sync(0xffffffffu, mbar_wait(bar.o_full(t), o_cnt & 1, abort_flag, p.status, p.wait_limit)))
            return;
        ++o_cnt;
        tc_fence_after();

        // Rows of this tile that hold a query row: a packed tile fills
        // heads * L of its 128 rows, a prefill tile ends at row L.
        const int n_valid = PK ? packed_rows(p, seg.h).heads * p.L : imin(kBlockQ, seg.L - q_tile0);
        const bool warp_live = (r & ~31) < n_valid;  // warp-uniform: tcgen05.ld is warp-collective
        const bool row_live = r < n_valid;

        // A later piece of a cut tile publishes its partial (unscaled
        // accumulator, row max, row sum of the live rows) for the finalizer; a
        // packed tile's finalizer publishes its own too and then merges them
        // all with the whole warpgroup (few live rows, many contributors).
        if (!ip.complete && (PK || !ip.finalizer)) {
            float *slot = p.partial + static_cast<size_t>(partial_slot(blockIdx.x, (PK && ip.finalizer) ? 1 : t)) *
                                          partial_slot_floats<D>();
            if (warp_live) {
#pragma unroll
                for (int cc = 0; cc < D / 32; ++cc) {
                    uint32_t o[32];
                    tmem_ld32(tO + cc * 32, o);
                    float4 *dst = reinterpret_cast<float4 *>(slot + r * D + cc * 32);
                    if (row_live) {
#pragma unroll
                        for (int v4 = 0; v4 < 8; ++v4)
                            __stcg(dst + v4,
                                   make_float4(__uint_as_float(o[4 * v4]), __uint_as_float(o[4 * v4 + 1]),
                                               __uint_as_float(o[4 * v4 + 2]), __uint_as_float(o[4 * v4 + 3])));
                    }
                }
                if (row_live) {
                    __stcg(slot + 128 * D + r, m_ref);
                    __stcg(slot + 128 * D + 128 + r, l);
                }
            }
            if (PK && ip.finalizer) {
                if (!merge_packed<D, MODE>(p, seg, sp, n_valid, epoch, abort_flag, bar, merge_steps)) return;
                continue;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(bar.pub(t));
            if (r == 0 && mbar_wait(bar.pub(t), pub_cnt & 1, abort_flag, p.status, p.wait_limit)) {
                __threadfence();
                st_release_gpu(p.ready + partial_slot(blockIdx.x, t), epoch);
            }
            ++pub_cnt;
            continue;
        }

        // Finalizer of a cut tile: merge the partials of the CTAs that hold
        // the rest of its key range (tiny-llm Week 2 Day 5, Task 1 merge:
        // m* = max m_k, l* = sum e^(m_k - m*) l_k, a* = sum e^(m_k - m*) a_k).
        float f_own = 1.f, m_star = m_ref;
        int c_last = blockIdx.x;
        if (!ip.complete) {
            c_last = last_contributor(p.W, gridDim.x, blockIdx.x, seg, sp, t);
            if (r == 0) {
                bool ok = true;
                for (int k = blockIdx.x + 1; k <= c_last && ok; ++k)
                    ok = flag_wait(p.ready + partial_slot(k, t), epoch, abort_flag, p.status, p.wait_limit);
                mbar_arrive(bar.fin(t));  // arrive even on failure; the abort flag tells
            }
            if (!__all_sync(0xffffffffu, mbar_wait(bar.fin(t), fin_cnt & 1, abort_flag, p.status, p.wait_limit)))
                return;
            ++fin_cnt;
            if (*abort_flag) return;
            if (row_live) {
#pragma unroll 4
                for (int k = blockIdx.x + 1; k <= c_last; ++k)
                    m_star = fmaxf(m_star, __ldcg(p.partial + static_cast<size_t>(partial_slot(k, t)) *
                                                                  partial_slot_floats<D>() + 128 * D + r));
                f_own = (m_ref == -CUDART_INF_F) ? 0.f : ex2((m_ref - m_star) * c);
                l *= f_own;
#pragma unroll 4
                for (int k = blockIdx.x + 1; k <= c_last; ++k) {
                    const float *slot = p.partial + static_cast<size_t>(partial_slot(k, t)) * partial_slot_floats<D>();
                    const float mk = __ldcg(slot + 128 * D + r);
                    const float fk = (mk == -CUDART_INF_F) ? 0.f : ex2((mk - m_star) * c);
                    l = fmaf(fk, __ldcg(slot + 128 * D + 128 + r), l);
                }
            }
        }

        // Final FP32 normalisation, then BF16 (a row with no allowed key has
        // l == 0 and is written as zeros).
        if (!warp_live) continue;
        if (row_live) l = add_sink(p, l, m_star, c, out_head);  // m_star == m_ref for a whole tile
        if (MODE == kModeLse && row_valid)
            p.lse[static_cast<size_t>(seg.b * p.Hq + out_head) * p.L + row] =
                l > 0.f ? fmaf(m_star, c, __log2f(l)) : CUDART_INF_F;
        const float inv = l > 0.f ? 1.f / l : 0.f;
        __nv_bfloat16 *orow = nullptr;
        if (row_valid)  // dense [B,Hq,L,D]; varlen packed [total_q, Hq, D]
            orow = p.o + (LY == kLayoutVarlen ? static_cast<size_t>(seg.q_base + row) * p.Hq + out_head
                                   : static_cast<size_t>(seg.b * p.Hq + out_head) * p.L + row) *
                             static_cast<size_t>(D);
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) {
            uint32_t o[32];
            tmem_ld32(tO + cc * 32, o);
            if (!ip.complete && row_live) {
#pragma unroll
                for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * f_own);
#pragma unroll 2
                for (int k = blockIdx.x + 1; k <= c_last; ++k) {
                    const float *slot = p.partial + static_cast<size_t>(partial_slot(k, t)) * partial_slot_floats<D>();
                    const float mk = __ldcg(slot + 128 * D + r);
                    const float fk = (mk == -CUDART_INF_F) ? 0.f : ex2((mk - m_star) * c);
                    const float4 *src = reinterpret_cast<const float4 *>(slot + r * D + cc * 32);
#pragma unroll
                    for (int v4 = 0; v4 < 8; ++v4) {
                        const float4 a = __ldcg(src + v4);
                        o[4 * v4] = __float_as_uint(fmaf(fk, a.x, __uint_as_float(o[4 * v4])));
                        o[4 * v4 + 1] = __float_as_uint(fmaf(fk, a.y, __uint_as_float(o[4 * v4 + 1])));
                        o[4 * v4 + 2] = __float_as_uint(fmaf(fk, a.z, __uint_as_float(o[4 * v4 + 2])));
                        o[4 * v4 + 3] = __float_as_uint(fmaf(fk, a.w, __uint_as_float(o[4 * v4 + 3])));
                    }
                }
            }
            uint32_t w[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
                w[i] = pack_bf16(__uint_as_float(o[2 * i]) * inv, __uint_as_float(o[2 * i + 1]) * inv);
            if (orow) {
                uint4 *dst = reinterpret_cast<uint4 *>(orow + cc * 32);
#pragma unroll
                for (int v4 = 0; v4 < 4; ++v4)
                    dst[v4] = make_uint4(w[4 * v4], w[4 * v4 + 1], w[4 * v4 + 2], w[4 * v4 + 3]);
            }
        }
    }
#ifdef TFA_TRACE
    if (threadIdx.x == 0 && blockIdx.x < 1024) g_tfa_cta_time[blockIdx.x][2] = globaltimer_ns();
#endif
}

// ------------------------------------------------------------------ kernel
template <int D, bool KM, int MODE, int LY, bool PK>
__global__ void __launch_bounds__(kThreads, 1)
    tfa_prefill_kernel(const __grid_constant__ CUtensorMap tm_q,
                       const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const Params p) {
    using C = Cfg<D>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t sbase = (raw + 1023u) & ~1023u;  // 128-byte swizzle wants 1 KB alignment
    uint8_t *gbase = smem_raw + (sbase - raw);
    Bars bar{sbase + C::kBarOff, C::kSlots};
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(gbase + C::kMiscOff);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(gbase + C::kMiscOff + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int t = 0; t < 2; ++t) {
            mbar_init(bar.q_full(t), 1);
            mbar_init(bar.q_empty(t), 1);
            mbar_init(bar.s_full(t), 1);
            mbar_init(bar.p_full(t), 4);
            mbar_init(bar.o_full(t), 1);
        }
        for (int s = 0; s < C::kSlots; ++s) {
            mbar_init(bar.kv_full(s), 1);
            mbar_init(bar.kv_empty(s), 1);
        }
        mbar_init(bar.done(), 1);
        for (int t = 0; t < 2; ++t) {
            mbar_init(bar.pub(t), 4);
            mbar_init(bar.fin(t), 1);
            mbar_init(bar.p_part(t), 4);
        }
        mbar_init(bar.merge_step(), 4);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(smem_addr(tmem_slot), C::kTmemCols);
        tmem_relinquish();
    }
    if (KM && warp == 8) {
        // ones block (column 0 = 1.0) and all-zero bias blocks; the load warp
        // later rewrites only the bias blocks' column 0
        uint32_t *z = reinterpret_cast<uint32_t *>(gbase + C::kBiasOff);
        for (int i = lane; i < (C::kSlots + 1) * C::kBiasBytes / 4; i += 32) z[i] = 0u;
        __syncwarp();
        for (int n = lane; n < 128; n += 32)
            *reinterpret_cast<uint16_t *>(gbase + C::kOnesOff + bias_offset(n, 0)) = 0x3F80u;
        fence_proxy_async_smem();
    }
    if (LY == kLayoutVarlen && warp < 8) {
        // validated copy of cu_seqlens; a bad sequence is skipped and reported
        int *tab = reinterpret_cast<int *>(gbase + C::kTableOff);
        for (int b = threadIdx.x; b < p.B; b += 256) {
            const int q0 = __ldg(p.cu_q + b), q1 = __ldg(p.cu_q + b + 1);
            const int k0 = __ldg(p.cu_k + b), k1 = __ldg(p.cu_k + b + 1);
            const bool ok = q0 >= 0 && q1 >= q0 && q1 <= p.total_q && k0 >= 0 && k1 >= k0 &&
                            k1 <= p.total_k && q1 - q0 <= p.shape.L && (!p.causal || k1 - k0 >= q1 - q0);
            tab[b] = q0;
            tab[kMaxVarlenSeqs + b] = ok ? q1 - q0 : 0;
            tab[2 * kMaxVarlenSeqs + b] = k0;
            tab[3 * kMaxVarlenSeqs + b] = k1 - k0;
            if (!ok && blockIdx.x == 0) atomicOr(p.status, TFA_DEVICE_BAD_SEQLENS);
        }
    }
    if (LY == kLayoutVarlen && p.shape.n_qp <= kMaxVarlenGroups) {
        // The compact deal (the same in every CTA): sequences sorted by their
        // item groups (query-tile pairs; query tiles with head pairs), longest
        // first, by a bitonic sort of unique keys (groups << 10 | 1023 - b)
        // over all threads, then per group the items that exist and their
        // prefix sums.  Without it a CTA's share of the item grid would hold
        // empty slots where short sequences end.
        __syncthreads();  // the table is complete
        const int *tab = reinterpret_cast<const int *>(gbase + C::kTableOff);
        unsigned *order = reinterpret_cast<unsigned *>(gbase + C::kOrderOff);
        int *gstart = reinterpret_cast<int *>(gbase + C::kGroupStartOff);
        int n = 1;
        while (n < p.B) n <<= 1;
        for (int i = threadIdx.x; i < n; i += kThreads) {
            const int rows = p.shape.hp ? kBlockQ : 2 * kBlockQ;  // query rows per item group
            const int pairs = i < p.B ? (tab[kMaxVarlenSeqs + i] + rows - 1) / rows : 0;
            order[i] = i < p.B ? (static_cast<unsigned>(pairs) << 10) | static_cast<unsigned>(1023 - i) : 0u;
        }
        __syncthreads();
        for (int k = 2; k <= n; k <<= 1) {
            for (int j = k >> 1; j > 0; j >>= 1) {
                for (int i = threadIdx.x; i < n; i += kThreads) {
                    const int l = i ^ j;
                    if (l > i) {
                        const unsigned a = order[i], b = order[l];
                        if ((i & k) == 0 ? a < b : a > b) {  // decreasing overall
                            order[i] = b;
                            order[l] = a;
                        }
                    }
                }
                __syncthreads();
            }
        }
        const int n_qp = p.shape.n_qp;
        for (int rr = threadIdx.x; rr < n_qp; rr += kThreads) {
            // sequences with item group qp: those with more than qp groups
            const unsigned bound = static_cast<unsigned>(group_qp(p.shape, rr) + 1) << 10;
            int lo = 0, hi = p.B;
            while (lo < hi) {
                const int mid = (lo + hi) >> 1;
                if (order[mid] >= bound) lo = mid + 1;
                else hi = mid;
            }
            gstart[rr + 1] = lo * p.shape.Hq;  // items per sequence: its (virtual) heads
        }
        if (threadIdx.x == 0) gstart[0] = 0;
        __syncthreads();
        if (warp == 0) {  // prefix sums over the groups, a chunk per lane
            const int per = (n_qp + 31) / 32;
            const int a0 = 1 + lane * per, a1 = imin(a0 + per, n_qp + 1);
            int sum = 0;
            for (int i = a0; i < a1; ++i) sum += gstart[i];
            int incl = sum;
#pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, incl, d);
                if (lane >= d) incl += y;
            }
            int run = incl - sum;
            for (int i = a0; i < a1; ++i) {
                run += gstart[i];
                gstart[i] = run;
            }
        }
    }
    if (warp == 8 && lane == 0) {
        prefetch_tensormap(&tm_q);
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
#ifdef TFA_TRACE
    if (threadIdx.x == 0 && blockIdx.x < 1024) g_tfa_cta_time[blockIdx.x][0] = globaltimer_ns();
#endif

    if (warp < 8) {
        reg_alloc<kRegsSoftmax>();
        softmax_role<D, KM, MODE, LY, PK>(p, warp >> 2, tmem, bar, abort_flag);
    } else {
        reg_dealloc<kRegsOther>();
        if (warp == 8 && (lane == 0 || KM))
            load_role<D, KM, LY, PK>(p, &tm_q, &tm_k, &tm_v, sbase, gbase, bar, abort_flag);
        if (warp == 9 && lane == 0) mma_role<D, KM, LY, PK>(p, sbase, tmem, bar, abort_flag);
    }

    tc_fence_before();
    __syncthreads();
#ifdef TFA_TRACE
    if (threadIdx.x == 0 && blockIdx.x < 1024) g_tfa_cta_time[blockIdx.x][1] = globaltimer_ns();
#endif
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
    // The last CTA to finish advances the epoch for the next launch; every
    // CTA read it before arriving here, and launches on a stream do not overlap.
    if (p.ctl && threadIdx.x == 0) {
        __threadfence();
        if (atomicAdd(p.ctl + 1, 1u) == gridDim.x - 1) {
            atomicExch(p.ctl + 1, 0u);
            atomicAdd(p.ctl, 1u);
        }
    }
}

}  // namespace tfa
