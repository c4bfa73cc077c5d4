// tfa_plan.h -- work enumeration for tiled GQA prefill attention, shared by the
// sm_100a kernel (device) and tfa_plan_qtile (host), so the host-side tests
// check the exact arithmetic the kernel runs.
//
// A 128-row query tile covers new rows [q0, qe) (qe = min(q0 + 128, L)), i.e.
// absolute positions [P + q0, P + qe - 1] with P = S - L.  It visits the
// 128-key tiles from kt_lo to kt_hi: the first tile holding a key that some row
// may see under the sliding window, and the last tile holding a key that the
// last row may see under the causal mask.  Tiles outside that band hold no
// allowed (row, key) pair and are skipped without loading K/V -- the banded
// prefill of mlx-lm PR "Skip fully masked key tiles in Flint sliding-window
// prefill", and brotensor flash_attention_decode_masked's "fully masked key
// tiles are skipped without touching K/V".  Inside the band, only tiles that
// cross the causal diagonal, the window's lower edge, the key tail (S) or that
// carry a key mask evaluate the mask predicate; interior tiles skip it.
#pragma once

#define TFA_HD __host__ __device__ __forceinline__

namespace tfa {

constexpr int kBlockQ = 128;
constexpr int kBlockK = 128;
constexpr unsigned kFlagNoTileSkip = 1u;
constexpr unsigned kFlagMaskAll = 2u;

struct KeyRange {
    int lo, hi;
};

TFA_HD int imin(int a, int b) { return a < b ? a : b; }
TFA_HD int imax(int a, int b) { return a > b ? a : b; }

TFA_HD KeyRange qtile_key_range(int L, int S, int causal, int window, int q0, unsigned flags) {
    const int P = S - L;
    const int qe = imin(q0 + kBlockQ, L);
    KeyRange r;
    r.hi = causal ? (P + qe - 1) / kBlockK : (S - 1) / kBlockK;
    r.lo = 0;
    if (causal && window > 0) {
        const int first_key = P + q0 - window + 1;  // lowest key the first row may see
        r.lo = first_key > 0 ? first_key / kBlockK : 0;
    }
    if (flags & kFlagNoTileSkip) {
        r.lo = 0;
        r.hi = (S - 1) / kBlockK;
    }
    return r;
}

TFA_HD bool key_tile_needs_mask(int L, int S, int causal, int window, int has_key_mask, int q0,
                                int kt, unsigned flags) {
    if (has_key_mask || (flags & kFlagMaskAll)) return true;
    const int P = S - L;
    const int qe = imin(q0 + kBlockQ, L);
    const int k0 = kt * kBlockK;
    const int k1 = k0 + kBlockK - 1;
    if (k1 >= S) return true;                                         // key tail
    if (causal && k1 > P + q0) return true;                           // crosses the diagonal
    if (causal && window > 0 && k0 <= P + qe - 1 - window) return true;  // crosses window edge
    return false;
}

// The query tiles that hold a row seeing some key of 128-key tile kt (the
// transpose of qtile_key_range, for the backward pass that walks key tiles):
// a row i sees key j iff (causal => j <= P + i) and (window => j > P + i - W).
// Returns lo > hi when no row sees the tile.
TFA_HD KeyRange ktile_query_range(int L, int S, int causal, int window, int kt) {
    const int P = S - L;
    const int k0 = kt * kBlockK;
    const int k1 = imin(k0 + kBlockK - 1, S - 1);
    const int nqt = (L + kBlockQ - 1) / kBlockQ;
    KeyRange r;
    r.lo = 0;
    r.hi = nqt - 1;
    if (causal) {
        const int first_row = k0 - P;  // the first row that sees key k0
        if (first_row > L - 1) {
            r.lo = 1;
            r.hi = 0;
            return r;
        }
        r.lo = first_row > 0 ? first_row / kBlockQ : 0;
        if (window > 0) {
            const int last_row = k1 - P + window - 1;  // the last row that sees key k1
            if (last_row < 0) {
                r.lo = 1;
                r.hi = 0;
                return r;
            }
            r.hi = imin(last_row, L - 1) / kBlockQ;
        }
    }
    return r;
}

}  // namespace tfa
