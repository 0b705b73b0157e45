// Gate normalisation, per-query Top-K threshold selection, and the per-q-tile
// union of selected blocks used by the tensor-core kernels.
//
// SAS paper (arXiv 2609.13141): §4.1 eq. 4 and §4.2 eq. 6 (softmax gates in log
// form over the historical blocks), §4.3 "Kernel Design" and Appendix E (Top-K
// realised as a per-query threshold on the log gate, no sort).
#include "sas_common.cuh"
#include "sas_kernels.h"

namespace sas {

// ---------------------------------------------------------------------------
// logG[row, m] = s[row, m] - LSE(s[row, :c]) for m < c, -inf otherwise.
// One warp per (b, g, t) row; two passes over the row (max, then sum of exp).
// HBM-bound: reads the causal part of s once, writes the full logG row once.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) gate_normalize_kernel(const float* __restrict__ s, float* __restrict__ logG,
                                                             long long rows, int T, int NB) {
  const int lane = threadIdx.x & 31;
  const long long row = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= rows) return;
  const int t = (int)(row % T);
  const int c = min(t / kBlock, NB);
  const float* src = s + row * (long long)NB;
  float* dst = logG + row * (long long)NB;
  float mx = -INFINITY;
  for (int m = lane; m < c; m += 32) mx = fmaxf(mx, __ldg(src + m));
#pragma unroll
  for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  float sum = 0.f;
  for (int m = lane; m < c; m += 32) sum += expf(__ldg(src + m) - mx);
#pragma unroll
  for (int o = 16; o; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  const float lse = mx + logf(sum);
  for (int m = lane; m < NB; m += 32) dst[m] = (m < c) ? (__ldg(src + m) - lse) : -INFINITY;
}

// Threshold (tau, tau_idx) and optional ascending index list of one row whose
// keys are in KREG registers per lane (key of block m = lane + 32 i in keys[i]).
// Block indices written (tau_idx, the list) are base + the key's position.
template <int KREG>
__device__ __forceinline__ void select_keys_regs(const uint32_t (&keys)[KREG], int c, int H, uint32_t* hist,
                                                 float* tau_out, int32_t* tidx_out, int32_t* out, int base = 0) {
  const int lane = threadIdx.x & 31;
  uint32_t tkey = 0u, asc = 0u;
  int tidx = -1;
  // Budgets up to 16 blocks: the threshold from the lanes' largest keys, and the
  // ascending list (when requested) by a second warp sort of the 32 candidates.
  if (H <= 16 && pivot_select_keys(keys, c, H, reinterpret_cast<uint2*>(hist), &tkey, &tidx, out ? &asc : nullptr)) {
    if (lane == 0) {
      *tau_out = key_float(tkey);
      *tidx_out = base + tidx;
    }
    if (out && lane < H) out[lane] = base + (int32_t)asc;   // exactly H blocks, ascending
    return;
  }
  // Larger budgets: the threshold from the lanes' two largest keys when that
  // bounds it, else the bisection; the ascending list (when requested) then by a
  // ballot over the row's keys in block order.
  if (!(H > 16 && H <= 63 && pivot2_select_keys(keys, c, H, reinterpret_cast<uint2*>(hist), &tkey, &tidx))) {
    int take_eq = 0;
    tkey = radix_select_keys(keys, c, H, nullptr, &take_eq);
    tidx = tie_index_keys(keys, c, tkey, take_eq);
  }
  if (lane == 0) {
    *tau_out = key_float(tkey);
    *tidx_out = base + tidx;
  }
  if (out) {
    int pos = 0;
#pragma unroll
    for (int i = 0; i < KREG; ++i) {
      if (32 * i >= c) break;
      const int m = lane + 32 * i;
      const bool take = m < c && (keys[i] > tkey || (keys[i] == tkey && m <= tidx));
      const uint32_t bal = __ballot_sync(0xffffffffu, take);
      if (take) out[pos + __popc(bal & ((1u << lane) - 1u))] = base + m;
      pos += __popc(bal);
    }
    for (int k = pos + lane; k < H; k += 32) out[k] = -1;
  }
}

template <int KREG>
__device__ __forceinline__ void select_row_regs(const float* __restrict__ v, int c, int H, uint32_t* hist,
                                                float* tau_out, int32_t* tidx_out, int32_t* out) {
  uint32_t keys[KREG];
  load_row_keys(v, c, keys);
  select_keys_regs(keys, c, H, hist, tau_out, tidx_out, out);
}

// Rows that select nothing or everything: (+inf, -1) / (-inf, c-1) and the list.
__device__ __forceinline__ bool select_trivial_row(int c, int H, float* tau_out, int32_t* tidx_out, int32_t* out) {
  const int lane = threadIdx.x & 31;
  if (min(c, H) == 0) {
    if (lane == 0) {
      *tau_out = INFINITY;
      *tidx_out = -1;
    }
    if (out)
      for (int k = lane; k < H; k += 32) out[k] = -1;
    return true;
  }
  if (c <= H) {
    if (lane == 0) {
      *tau_out = -INFINITY;
      *tidx_out = c - 1;
    }
    if (out)
      for (int k = lane; k < H; k += 32) out[k] = (k < c) ? k : -1;
    return true;
  }
  return false;
}

__global__ void __launch_bounds__(256) select_threshold_kernel(const float* __restrict__ logG, float* __restrict__ tau,
                                                               int32_t* __restrict__ tau_idx,
                                                               int32_t* __restrict__ sel, long long rows, int T,
                                                               int NB, int H) {
  __shared__ __align__(16) uint32_t hist_all[8][256];   // per-warp scratch of the select
  const int lane = threadIdx.x & 31;
  const int wid = threadIdx.x >> 5;
  const long long row = (long long)blockIdx.x * 8 + wid;
  if (row >= rows) return;
  const int t = (int)(row % T);
  const int c = min(t / kBlock, NB);
  const float* v = logG + row * (long long)NB;
  int32_t* out = sel ? sel + row * (long long)H : nullptr;
  if (select_trivial_row(c, H, tau + row, tau_idx + row, out)) return;
  if (c <= 32 * kSelectReg) {
    // Keys in registers: one read of the row; the threshold, the tie index and
    // the index list all work on them (register width picked by row length).
    if (c <= 128)
      select_row_regs<4>(v, c, H, hist_all[wid], tau + row, tau_idx + row, out);
    else if (c <= 256)
      select_row_regs<8>(v, c, H, hist_all[wid], tau + row, tau_idx + row, out);
    else if (c <= 512)
      select_row_regs<16>(v, c, H, hist_all[wid], tau + row, tau_idx + row, out);
    else
      select_row_regs<32>(v, c, H, hist_all[wid], tau + row, tau_idx + row, out);
    return;
  }
  int take_eq = 0;
  const uint32_t tkey = radix_select_global(v, c, H, hist_all[wid], &take_eq);
  const int tidx = tie_index_global(v, c, tkey, take_eq);
  if (lane == 0) {
    tau[row] = key_float(tkey);
    tau_idx[row] = tidx;
  }
  if (out) {
    int pos = 0;
    for (int base = 0; base < c; base += 32) {
      const int m = base + lane;
      bool take = false;
      if (m < c) {
        const uint32_t k = float_key(v[m]);
        take = (k > tkey) || (k == tkey && m <= tidx);
      }
      const uint32_t bal = __ballot_sync(0xffffffffu, take);
      if (take) out[pos + __popc(bal & ((1u << lane) - 1u))] = m;
      pos += __popc(bal);
    }
    for (int k = pos + lane; k < H; k += 32) out[k] = -1;
  }
}

// ---------------------------------------------------------------------------
// Normalisation and selection in one pass (one warp per row, the row in
// registers): the same logG values as gate_normalize_kernel (same arithmetic,
// same summation order) written once, and the selection taken on them, so the
// outputs equal the two separate calls bit for bit. Rows longer than
// 32 * kSelectReg blocks use the two kernels.
// ---------------------------------------------------------------------------
// With lse_out set (compact gates) the row's LSE of s goes there and no logG is
// written (dst unused): consumers rebuild logG[m] = s[m] - LSE, the same fp32
// subtraction as here.
template <int KREG>
__device__ __forceinline__ void normalize_select_row(const float* __restrict__ src, float* __restrict__ dst, int c_lo,
                                                     int c, int NB, int H, uint32_t* hist, float* tau_out,
                                                     int32_t* tidx_out, int32_t* out, float* lse_out = nullptr) {
  // The row's historical blocks are c_lo .. c-1 (c_lo > 0 only for a later document of a packed sequence).
  const int lane = threadIdx.x & 31;
  const int n = c - c_lo;
  float v[KREG];
#pragma unroll
  for (int i = 0; i < KREG; ++i) v[i] = (lane + 32 * i < n) ? __ldg(src + c_lo + lane + 32 * i) : -INFINITY;
  float mx = -INFINITY;
#pragma unroll
  for (int i = 0; i < KREG; ++i) mx = fmaxf(mx, v[i]);
#pragma unroll
  for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  float sum = 0.f;
#pragma unroll
  for (int i = 0; i < KREG; ++i)
    if (lane + 32 * i < n) sum += expf(v[i] - mx);
#pragma unroll
  for (int o = 16; o; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  const float lse = mx + logf(sum);
  uint32_t keys[KREG];
#pragma unroll
  for (int i = 0; i < KREG; ++i) {
    const int q = lane + 32 * i;
    const float lg = (q < n) ? v[i] - lse : -INFINITY;
    if (!lse_out && c_lo + q < NB) dst[c_lo + q] = lg;
    keys[i] = (q < n) ? float_key(lg) : 0u;
    v[i] = lg;
  }
  if (lse_out) {
    if (lane == 0) *lse_out = lse;
  } else {
    for (int m = lane; m < c_lo; m += 32) dst[m] = -INFINITY;
    for (int m = c_lo + lane + 32 * KREG; m < NB; m += 32) dst[m] = -INFINITY;
  }
  if (c_lo == 0) {
    if (select_trivial_row(c, H, tau_out, tidx_out, out)) return;
  } else if (min(n, H) == 0 || n <= H) {
    // Nothing, or every block of the row's own document: the threshold is its
    // least gate (and the last block holding it), which keeps no block of an
    // earlier document (their gates are -inf).
    float tmin = INFINITY;
#pragma unroll
    for (int i = 0; i < KREG; ++i)
      if (lane + 32 * i < n) tmin = fminf(tmin, v[i]);
#pragma unroll
    for (int o = 16; o; o >>= 1) tmin = fminf(tmin, __shfl_xor_sync(0xffffffffu, tmin, o));
    int tix = -1;
#pragma unroll
    for (int i = 0; i < KREG; ++i)
      if (lane + 32 * i < n && v[i] == tmin) tix = lane + 32 * i;
#pragma unroll
    for (int o = 16; o; o >>= 1) tix = max(tix, __shfl_xor_sync(0xffffffffu, tix, o));
    const bool none = min(n, H) == 0;
    if (lane == 0) {
      *tau_out = none ? INFINITY : ((tmin == 0.f) ? 0.f : tmin);
      *tidx_out = none ? -1 : c_lo + tix;
    }
    if (out)
      for (int k = lane; k < H; k += 32) out[k] = (!none && k < n) ? c_lo + k : -1;
    return;
  }
  select_keys_regs(keys, n, H, hist, tau_out, tidx_out, out, c_lo);
}

// KREG from the row length NB on the host, so short rows run with few registers
// (and many warps per SM): the pivot select is instruction-bound.
template <int KREG>
__global__ void __launch_bounds__(256) normalize_select_kernel(const float* __restrict__ s, float* __restrict__ logG,
                                                               float* __restrict__ tau, int32_t* __restrict__ tau_idx,
                                                               int32_t* __restrict__ sel, long long rows, int T,
                                                               int NB, int H) {
  __shared__ __align__(16) uint32_t hist_all[8][256];   // per-warp scratch of the select
  const int wid = threadIdx.x >> 5;
  const long long row = (long long)blockIdx.x * 8 + wid;
  if (row >= rows) return;
  const int t = (int)(row % T);
  const int c = min(t / kBlock, NB);
  int32_t* out = sel ? sel + row * (long long)H : nullptr;
  normalize_select_row<KREG>(s + row * (long long)NB, logG + row * (long long)NB, 0, c, NB, H, hist_all[wid],
                             tau + row, tau_idx + row, out);
}

// Compact gates: the same per row, writing the LSE of the row's historical
// scores instead of the logG row.
template <int KREG>
__global__ void __launch_bounds__(256) normalize_select_compact_kernel(const float* __restrict__ s,
                                                                       float* __restrict__ lse,
                                                                       float* __restrict__ tau,
                                                                       int32_t* __restrict__ tau_idx,
                                                                       int32_t* __restrict__ sel, long long rows,
                                                                       int T, int NB, int H) {
  __shared__ __align__(16) uint32_t hist_all[8][256];   // per-warp scratch of the select
  const int wid = threadIdx.x >> 5;
  const long long row = (long long)blockIdx.x * 8 + wid;
  if (row >= rows) return;
  const int t = (int)(row % T);
  const int c = min(t / kBlock, NB);
  int32_t* out = sel ? sel + row * (long long)H : nullptr;
  normalize_select_row<KREG>(s + row * (long long)NB, nullptr, 0, c, NB, H, hist_all[wid], tau + row, tau_idx + row,
                             out, lse + row);
}

// Packed sequences: the same per row, over the blocks of the row's own document
// (its first block from the document table, by binary search; documents start
// on block boundaries).
template <int KREG>
__global__ void __launch_bounds__(256) normalize_select_varlen_kernel(
    const float* __restrict__ s, float* __restrict__ logG, float* __restrict__ tau, int32_t* __restrict__ tau_idx,
    int32_t* __restrict__ sel, long long rows, int T, int NB, int H, const DocTable docs) {
  __shared__ __align__(16) uint32_t hist_all[8][256];   // per-warp scratch of the select
  const int wid = threadIdx.x >> 5;
  const long long row = (long long)blockIdx.x * 8 + wid;
  if (row >= rows) return;
  const int t = (int)(row % T);
  const int cur = t / kBlock;
  int lo = 0, hi = docs.n - 1;   // the last document starting at or before block cur
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (docs.start_blk[mid] <= cur)
      lo = mid;
    else
      hi = mid - 1;
  }
  const int c = min(cur, NB);
  const int c_lo = min(docs.start_blk[lo], c);
  int32_t* out = sel ? sel + row * (long long)H : nullptr;
  normalize_select_row<KREG>(s + row * (long long)NB, logG + row * (long long)NB, c_lo, c, NB, H, hist_all[wid],
                             tau + row, tau_idx + row, out);
}

// ---------------------------------------------------------------------------
// Noisy selection for the "full*" training scope (SAS paper §4.1, Table 1 row
// 11: noise added to the scores before Top-K). One warp per row, the row in
// registers: the keys logG + noise (an fp32 add) give the Top-(K-1) set; logG_sel
// keeps logG on that set and -inf elsewhere, and (tau, tau_idx) is the threshold
// of logG_sel (the least kept gate and the last kept block holding it), so that
// the attention calls, which find the selected blocks by thresholding their gate
// tensor, find exactly this set in logG_sel. Blocks with a -inf gate (other
// documents of a packed sequence) are never chosen.
// ---------------------------------------------------------------------------
template <int KREG>
__global__ void __launch_bounds__(256) select_noisy_kernel(const float* __restrict__ logG,
                                                           const float* __restrict__ noise,
                                                           float* __restrict__ logG_sel, float* __restrict__ tau,
                                                           int32_t* __restrict__ tau_idx, int32_t* __restrict__ sel,
                                                           long long rows, int T, int NB, int H) {
  __shared__ __align__(16) uint32_t hist_all[8][256];   // per-warp scratch of the select
  const int lane = threadIdx.x & 31;
  const int wid = threadIdx.x >> 5;
  const long long row = (long long)blockIdx.x * 8 + wid;
  if (row >= rows) return;
  const int t = (int)(row % T);
  const int c = min(t / kBlock, NB);
  const float* lrow = logG + row * (long long)NB;
  const float* nrow = noise + row * (long long)NB;
  float* dst = logG_sel + row * (long long)NB;
  int32_t* out = sel ? sel + row * (long long)H : nullptr;
  // A block whose gate is -inf (another document of a packed sequence) is never a
  // candidate: its key is 0, below every real key.
  float lg[KREG];
  uint32_t keys[KREG];
  int n_fin = 0;
#pragma unroll
  for (int i = 0; i < KREG; ++i) {
    const int m = lane + 32 * i;
    lg[i] = (m < c) ? __ldg(lrow + m) : -INFINITY;
    const bool fin = lg[i] != -INFINITY;
    keys[i] = fin ? float_key(__fadd_rn(lg[i], __ldg(nrow + m))) : 0u;
    n_fin += fin ? 1 : 0;
  }
  n_fin = __reduce_add_sync(0xffffffffu, n_fin);
  bool take[KREG];
  if (min(n_fin, H) == 0 || n_fin <= H) {   // nothing, or every block with a gate
#pragma unroll
    for (int i = 0; i < KREG; ++i) take[i] = (H > 0) && lg[i] != -INFINITY;
  } else {
    uint32_t tk = 0u;
    int ti = -1;
    threshold_keys(keys, c, H, reinterpret_cast<uint2*>(hist_all[wid]), &tk, &ti);
#pragma unroll
    for (int i = 0; i < KREG; ++i) {
      const int m = lane + 32 * i;
      take[i] = m < c && keys[i] != 0u && (keys[i] > tk || (keys[i] == tk && m <= ti));
    }
  }
  // Threshold of logG_sel: the least kept gate and the last kept block holding it.
  float tmin = INFINITY;
#pragma unroll
  for (int i = 0; i < KREG; ++i)
    if (take[i]) tmin = fminf(tmin, lg[i]);
#pragma unroll
  for (int o = 16; o; o >>= 1) tmin = fminf(tmin, __shfl_xor_sync(0xffffffffu, tmin, o));
  int tix = -1;
#pragma unroll
  for (int i = 0; i < KREG; ++i)
    if (take[i] && lg[i] == tmin) tix = lane + 32 * i;
#pragma unroll
  for (int o = 16; o; o >>= 1) tix = max(tix, __shfl_xor_sync(0xffffffffu, tix, o));
  if (lane == 0) {
    if (min(n_fin, H) == 0) {
      tau[row] = INFINITY;
      tau_idx[row] = -1;
    } else if (n_fin == c && c <= H) {   // every historical block
      tau[row] = -INFINITY;
      tau_idx[row] = c - 1;
    } else {   // the least kept gate and the last kept block holding it
      tau[row] = (tmin == 0.f) ? 0.f : tmin;   // -0 and +0 are one threshold
      tau_idx[row] = tix;
    }
  }
#pragma unroll
  for (int i = 0; i < KREG; ++i) {
    const int m = lane + 32 * i;
    if (m < NB) dst[m] = take[i] ? lg[i] : -INFINITY;
  }
  for (int m = lane + 32 * KREG; m < NB; m += 32) dst[m] = -INFINITY;
  if (out) {
    int pos = 0;
#pragma unroll
    for (int i = 0; i < KREG; ++i) {
      const uint32_t bal = __ballot_sync(0xffffffffu, take[i]);
      if (take[i]) out[pos + __popc(bal & ((1u << lane) - 1u))] = lane + 32 * i;
      pos += __popc(bal);
    }
    for (int k = pos + lane; k < H; k += 32) out[k] = -1;
  }
}

// ---------------------------------------------------------------------------
// Selector-score gradient (SAS paper Appendix D.3, the softmax backward, with the
// gate gradient in log form): ds[m] = dLogG[m] - exp(logG[m]) * sum_{l<c} dLogG[l]
// for m < c_t, 0 otherwise. One warp per row; HBM-bound.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) gate_grad_kernel(const float* __restrict__ logG, const float* __restrict__ lse,
                                                        const float* __restrict__ dLogG, float* __restrict__ ds,
                                                        long long rows, int T, int NB) {
  const int lane = threadIdx.x & 31;
  const long long row = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= rows) return;
  const int t = (int)(row % T);
  const int c = min(t / kBlock, NB);
  const float* lg = logG + row * (long long)NB;
  const float* dl = dLogG + row * (long long)NB;
  float* out = ds + row * (long long)NB;
  float sum = 0.f;
  for (int m = lane; m < c; m += 32) sum += __ldg(dl + m);
#pragma unroll
  for (int o = 16; o; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  const float rl = (lse && c > 0) ? lse[row] : 0.f;   // raw scores: log g = s - LSE(s)
  for (int m = lane; m < NB; m += 32) out[m] = (m < c) ? __ldg(dl + m) - expf(__ldg(lg + m) - rl) * sum : 0.f;
}

// ---------------------------------------------------------------------------
// Union of the selected historical blocks over the rows of one q-tile (P
// consecutive positions of one (b, g); all G heads share the selection).
// masks[(bg * n_ptiles + pt) * NBW + w] bit i = block 32w + i is selected by
// at least one position of the tile (current blocks not included).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) tile_union_kernel(const float* __restrict__ logG, const float* __restrict__ lse,
                                                         const float* __restrict__ tau,
                                                         const int32_t* __restrict__ tau_idx,
                                                         uint32_t* __restrict__ masks, int T, int NB, int P,
                                                         int n_ptiles, int NBW) {
  extern __shared__ uint32_t words[];
  const int lane = threadIdx.x & 31;
  const int wid = threadIdx.x >> 5;
  const int nw = blockDim.x >> 5;
  const long long bg = blockIdx.x / n_ptiles;
  const int pt = blockIdx.x % n_ptiles;
  for (int w = threadIdx.x; w < NBW; w += blockDim.x) words[w] = 0u;
  __syncthreads();
  const int t0 = pt * P;
  for (int p = wid; p < P; p += nw) {
    const int t = t0 + p;
    if (t >= T) break;
    const long long row = bg * T + t;
    const int c = min(t / kBlock, NB);
    const float tv = tau[row];
    const int ti = tau_idx[row];
    const float* v = logG + row * (long long)NB;
    const float rl = (lse && c > 0) ? lse[row] : 0.f;   // raw scores: log g = s - LSE(s)
    for (int base = 0; base < c; base += 128) {   // four 32-block spans per round trip
      float x[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int m = base + 32 * u + lane;
        x[u] = (m < c) ? v[m] - rl : 0.f;
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int m = base + 32 * u + lane;
        const bool sel = m < c && ((x[u] > tv) || (x[u] == tv && m <= ti));
        const uint32_t bal = __ballot_sync(0xffffffffu, sel);
        if (lane == 0 && bal) atomicOr(&words[(base >> 5) + u], bal);
      }
    }
  }
  __syncthreads();
  uint32_t* dst = masks + ((long long)bg * n_ptiles + pt) * NBW;
  for (int w = threadIdx.x; w < NBW; w += blockDim.x) dst[w] = words[w];
}

// ------------------------------------------------------------------ launchers
cudaError_t launch_gate_normalize(const float* s, float* logG, long long rows, int T, int NB, cudaStream_t st) {
  const int warps = 8;
  const long long blocks = (rows + warps - 1) / warps;
  gate_normalize_kernel<<<(unsigned)blocks, warps * 32, 0, st>>>(s, logG, rows, T, NB);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_select_threshold(const float* logG, float* tau, int32_t* tau_idx, int32_t* sel, long long rows,
                                    int T, int NB, int H, cudaStream_t st) {
  const long long blocks = (rows + 7) / 8;
  select_threshold_kernel<<<(unsigned)blocks, 256, 0, st>>>(logG, tau, tau_idx, sel, rows, T, NB, H);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_normalize_select(const float* s, float* logG, float* tau, int32_t* tau_idx, int32_t* sel,
                                    long long rows, int T, int NB, int H, cudaStream_t st) {
  if (NB > 32 * kSelectReg) {   // rows longer than the registers hold: two passes
    cudaError_t e = launch_gate_normalize(s, logG, rows, T, NB, st);
    if (e != cudaSuccess) return e;
    return launch_select_threshold(logG, tau, tau_idx, sel, rows, T, NB, H, st);
  }
  const unsigned grid = (unsigned)((rows + 7) / 8);
  if (NB <= 128)
    normalize_select_kernel<4><<<grid, 256, 0, st>>>(s, logG, tau, tau_idx, sel, rows, T, NB, H);
  else if (NB <= 256)
    normalize_select_kernel<8><<<grid, 256, 0, st>>>(s, logG, tau, tau_idx, sel, rows, T, NB, H);
  else if (NB <= 512)
    normalize_select_kernel<16><<<grid, 256, 0, st>>>(s, logG, tau, tau_idx, sel, rows, T, NB, H);
  else
    normalize_select_kernel<kSelectReg><<<grid, 256, 0, st>>>(s, logG, tau, tau_idx, sel, rows, T, NB, H);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_normalize_select_varlen(const float* s, float* logG, float* tau, int32_t* tau_idx, int32_t* sel,
                                           long long rows, int T, int NB, int H, const DocTable& docs,
                                           cudaStream_t st) {
  const unsigned grid = (unsigned)((rows + 7) / 8);
  if (NB <= 128)
    normalize_select_varlen_kernel<4><<<grid, 256, 0, st>>>(s, logG, tau, tau_idx, sel, rows, T, NB, H, docs);
  else if (NB <= 256)
    normalize_select_varlen_kernel<8><<<grid, 256, 0, st>>>(s, logG, tau, tau_idx, sel, rows, T, NB, H, docs);
  else if (NB <= 512)
    normalize_select_varlen_kernel<16><<<grid, 256, 0, st>>>(s, logG, tau, tau_idx, sel, rows, T, NB, H, docs);
  else if (NB <= 32 * kSelectReg)
    normalize_select_varlen_kernel<kSelectReg><<<grid, 256, 0, st>>>(s, logG, tau, tau_idx, sel, rows, T, NB, H,
                                                                      docs);
  else
    return cudaErrorInvalidValue;
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_select_noisy(const float* logG, const float* noise, float* logG_sel, float* tau, int32_t* tau_idx,
                                int32_t* sel, long long rows, int T, int NB, int H, cudaStream_t st) {
  const unsigned grid = (unsigned)((rows + 7) / 8);
  if (NB <= 128)
    select_noisy_kernel<4><<<grid, 256, 0, st>>>(logG, noise, logG_sel, tau, tau_idx, sel, rows, T, NB, H);
  else if (NB <= 256)
    select_noisy_kernel<8><<<grid, 256, 0, st>>>(logG, noise, logG_sel, tau, tau_idx, sel, rows, T, NB, H);
  else if (NB <= 512)
    select_noisy_kernel<16><<<grid, 256, 0, st>>>(logG, noise, logG_sel, tau, tau_idx, sel, rows, T, NB, H);
  else if (NB <= 32 * kSelectReg)
    select_noisy_kernel<kSelectReg><<<grid, 256, 0, st>>>(logG, noise, logG_sel, tau, tau_idx, sel, rows, T, NB, H);
  else
    return cudaErrorInvalidValue;
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_normalize_select_compact(const float* s, float* lse, float* tau, int32_t* tau_idx, int32_t* sel,
                                            long long rows, int T, int NB, int H, cudaStream_t st) {
  const unsigned grid = (unsigned)((rows + 7) / 8);
  if (NB <= 128)
    normalize_select_compact_kernel<4><<<grid, 256, 0, st>>>(s, lse, tau, tau_idx, sel, rows, T, NB, H);
  else if (NB <= 256)
    normalize_select_compact_kernel<8><<<grid, 256, 0, st>>>(s, lse, tau, tau_idx, sel, rows, T, NB, H);
  else if (NB <= 512)
    normalize_select_compact_kernel<16><<<grid, 256, 0, st>>>(s, lse, tau, tau_idx, sel, rows, T, NB, H);
  else
    normalize_select_compact_kernel<kSelectReg><<<grid, 256, 0, st>>>(s, lse, tau, tau_idx, sel, rows, T, NB, H);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_gate_grad(const float* logG, const float* gate_lse, const float* dLogG, float* ds, long long rows,
                             int T, int NB, cudaStream_t st) {
  gate_grad_kernel<<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(logG, gate_lse, dLogG, ds, rows, T, NB);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_tile_union(const float* logG, const float* gate_lse, const float* tau, const int32_t* tau_idx,
                              uint32_t* masks, long long n_bg, int T, int NB, int P, int n_ptiles, int NBW,
                              cudaStream_t st) {
  const long long blocks = n_bg * n_ptiles;
  tile_union_kernel<<<(unsigned)blocks, 256, NBW * sizeof(uint32_t), st>>>(logG, gate_lse, tau, tau_idx, masks, T, NB,
                                                                           P, n_ptiles, NBW);
  count_launch();
  return cudaGetLastError();
}

}  // namespace sas
