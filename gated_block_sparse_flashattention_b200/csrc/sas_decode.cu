// SAS sparse decode step (memory-bound).
//
// SAS paper (arXiv 2609.13141) §4.3 Algorithm 2 (Top-K on the selector scores,
// then ungated attention over the current block and the selected blocks) and
// §5.1 "Inference implementation" (per-KV-group selection, GQA, gathering only
// the selected KV blocks).
//
// bf16 storage, contiguous cache, rows of up to 512 blocks and at least three
// (b, g) groups per four SMs: one kernel, decode_group_kernel, one CTA per
// (b, g) that selects, streams the group's blocks and writes o.
// Otherwise (paged caches, longer rows, fewer groups), three kernels:
//   decode_select_kernel    one warp (one CTA) per (b, g): Top-(K-1) of the score
//                           row; the attended list [c, selected blocks] goes to
//                           the workspace (rows over 1024 blocks:
//                           decode_select_radix_kernel, one 512-thread CTA per
//                           (b, g)); for a paged cache also each block's page.
//   decode_fused_mma_kernel persistent, two 4-warp CTAs per SM, each walking a
//                           contiguous run of items (b, g, attended block) with a
//                           3-stage TMA ring; the G heads' scores and P V run as
//                           m16n8k16 MMAs (fp32 accumulation); the items of one
//                           (b, g) are folded online and leave one fp32 partial.
//   decode_merge_kernel<S>  one CTA per (b, g): merges the partials into o.
// The second and third are programmatic dependents of the one before them.
// fp32 storage: decode_select_kernel, then decode_attn_kernel<float> (one
// 128-thread CTA per item on the CUDA cores, one bulk copy each for K and V),
// whose CTA taking the last ticket of a (b, g) merges its partials.
#include <algorithm>
#include <cudaTypedefs.h>

#include <mutex>

#include "sas_common.cuh"
#include "sas_kernels.h"
#include "sas_tmap.h"

namespace sas {
namespace decode {

constexpr int D = 128;
constexpr int ATT_THREADS = 128;         // attention CTA: 4 warps x 16 keys
constexpr int HC = 4;                    // heads per register chunk

struct Params {
  const void* q;
  const void* Kc;
  const void* Vc;
  const int32_t* seqlen;
  const float* s;
  void* o;
  int32_t* sel_out;
  int32_t* status;     // device status word (first word of the workspace)
  int32_t* att;        // [B*Hkv][K] attended blocks: [current, selected ascending], -1 padded
  float* lse_gate;     // [B*Hkv] log-sum-exp of the historical scores (log-gate option)
  int32_t* att_z;      // [B*Hkv][K] paged cache: plane (page * Hkv + g) of each attended block, -1 none
  const int32_t* page_table;   // [B][max_pages] page of each logical block (null: contiguous cache)
  int32_t* tickets;    // [B*Hkv] (fp32 attention kernel)
  int32_t* work;       // a counter the select kernel clears (unused by the current kernels)
  float* part_ml;      // [B*Hkv][n_slots][G][2]
  float* part_o;       // [B*Hkv][n_slots][G][D]
  int B, Hq, Hkv, Lmax, NBmax, K, apply_log_gate, G;
  int max_pages, num_pages;   // paged cache only
  int n_slots;         // partial slots per (b, g)
  float sm_scale;
};

template <typename T>
__device__ __forceinline__ float to_f(T v);
template <>
__device__ __forceinline__ float to_f<float>(float v) {
  return v;
}
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 v) {
  return __bfloat162float(v);
}

__device__ __forceinline__ void bulk_copy_g2s(uint32_t dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

// Programmatic dependent launch: the dependent grid may start once every CTA of
// this grid has called launch_dependents; its griddepcontrol.wait returns when
// this grid has completed and its memory operations are visible.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;"); }

// ---------------------------------------------------------------------------- selection
// Emits the H largest of n keys held in registers (position q = lane + 32 i in
// keys[i]; ties toward the lower position) as the list out[0..) of idx(q) in
// ascending q, also to so[0..) when requested; returns how many (min(n, H)).
// idx must be increasing in q, so the list is ascending in idx too. Warp-collective.
template <int KREG, typename Idx>
__device__ __forceinline__ int select_keys_list(const uint32_t (&keys)[KREG], int n, int H, uint2* cand, Idx idx,
                                                int32_t* out, int32_t* so) {
  const int lane = threadIdx.x & 31;
  if (n <= H) {   // every key
#pragma unroll
    for (int i = 0; i < KREG; ++i) {
      const int q = lane + 32 * i;
      if (q < n) {
        const int v = idx(q);
        out[q] = v;
        if (so) so[q] = v;
      }
    }
    return n;
  }
  uint32_t tk = 0u, asc = 0u;
  int tidx = -1;
  if (H <= 32 && pivot_select_keys(keys, n, H, cand, &tk, &tidx, &asc)) {
    if (lane < H) {
      const int v = idx((int)asc);
      out[lane] = v;
      if (so) so[lane] = v;
    }
    return H;
  }
  int take_eq = 0;
  tk = radix_select_keys(keys, n, H, nullptr, &take_eq);
  tidx = tie_index_keys(keys, n, tk, take_eq);
  int cnt = 0;
#pragma unroll
  for (int i = 0; i < KREG; ++i) {
    if (32 * i >= n) break;
    const int q = lane + 32 * i;
    const bool take = q < n && (keys[i] > tk || (keys[i] == tk && q <= tidx));
    const uint32_t bal = __ballot_sync(0xffffffffu, take);
    if (take) {
      const int lp = cnt + __popc(bal & ((1u << lane) - 1u));
      const int v = idx(q);
      out[lp] = v;
      if (so) so[lp] = v;
    }
    cnt += __popc(bal);
  }
  return cnt;
}

struct IdentityIdx {
  __device__ int operator()(int q) const { return q; }
};

// Emits the selected blocks of one score row (keys in registers) as the ascending
// list att[1..] (and so[0..] when requested); returns how many.
template <int KREG>
__device__ __forceinline__ int decode_select_row(const float* __restrict__ srow, int c, int H, int mode, uint2* cand,
                                                 int32_t* att, int32_t* so) {
  const int lane = threadIdx.x & 31;
  if (mode == 1) {   // every historical block
    for (int m = lane; m < c; m += 32) {
      att[1 + m] = m;
      if (so) so[m] = m;
    }
    return c;
  }
  uint32_t keys[KREG];
  load_row_keys(srow, c, keys);
  return select_keys_list(keys, c, H, cand, IdentityIdx{}, att + 1, so);
}

// Paged cache: the plane (page * Hkv + g) of every attended block of (b, g) for
// the attention kernel's copies. A page outside 0..num_pages-1 is reported as a
// bounds error and its block dropped from the list. Warp-collective; the warp
// wrote att itself (visible to its lanes after the __syncwarp).
__device__ __forceinline__ void map_pages(const Params& p, int bg, int32_t* att) {
  const int lane = threadIdx.x & 31;
  __syncwarp();
  const int b = bg / p.Hkv, g = bg % p.Hkv;
  int32_t* z = p.att_z + (long long)bg * p.K;
  for (int k = lane; k < p.K; k += 32) {
    const int m = att[k];
    int zz = -1;
    if (m >= 0) {
      const int pg = (m < p.max_pages) ? __ldg(p.page_table + (long long)b * p.max_pages + m) : -1;
      if (pg < 0 || pg >= p.num_pages) {
        set_status(p.status, SAS_DEV_ERR_BOUNDS);
        att[k] = -1;
      } else {
        zz = pg * p.Hkv + g;
      }
    }
    z[k] = zz;
  }
}

// Selected blocks of one score row (c historical blocks, mode as below) as the
// ascending list att[1..] (and so[0..] when requested); returns how many. Warp-
// collective. `scratch` is 256 words of this warp's shared memory (16-byte aligned).
// mode 0: nothing selected; 1: every historical block; 2: threshold.
__device__ __forceinline__ int select_row(const float* __restrict__ srow, int c, int H, int mode, uint32_t* scratch,
                                          int32_t* att, int32_t* so) {
  const int lane = threadIdx.x & 31;
  uint2* cand = reinterpret_cast<uint2*>(scratch);
  if (mode == 0) return 0;
  if (c <= 128) return decode_select_row<4>(srow, c, H, mode, cand, att, so);
  if (c <= 256) return decode_select_row<8>(srow, c, H, mode, cand, att, so);
  if (c <= 512) return decode_select_row<16>(srow, c, H, mode, cand, att, so);
  if (c <= 32 * kSelectReg) return decode_select_row<kSelectReg>(srow, c, H, mode, cand, att, so);
  uint32_t tk = 0u;
  int tidx = -1;
  if (mode == 2) {
    int take_eq = 0;
    tk = radix_select_global(srow, c, H, scratch, &take_eq);
    tidx = tie_index_global(srow, c, tk, take_eq);
  }
  int pos = 0;
  for (int base = 0; base < c; base += 32) {
    const int m = base + lane;
    bool take = false;
    if (m < c) {
      const uint32_t key = float_key(srow[m]);
      take = mode == 1 || (key > tk) || (key == tk && m <= tidx);
    }
    const uint32_t bal = __ballot_sync(0xffffffffu, take);
    if (take) {
      const int lp = pos + __popc(bal & ((1u << lane) - 1u));
      att[1 + lp] = m;
      if (so) so[lp] = m;
    }
    pos += __popc(bal);
  }
  return pos;
}

// log sum_{m < c} exp(s[m]) of one score row (the log-gate option); warp-collective.
__device__ __forceinline__ float row_lse(const float* __restrict__ srow, int c) {
  const int lane = threadIdx.x & 31;
  float mx = -INFINITY;
  for (int m = lane; m < c; m += 32) mx = fmaxf(mx, srow[m]);
#pragma unroll
  for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  float sum = 0.f;
  for (int m = lane; m < c; m += 32) sum += expf(srow[m] - mx);
#pragma unroll
  for (int o = 16; o; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  return (c > 0) ? mx + logf(sum) : 0.f;
}

// One warp (one CTA) per (b, g), so the rows spread over the SMs. KREG (from
// the score-row length NBmax) lets the row be loaded before the sequence length
// is known, so the two loads are in flight together; KREG = 0 is the generic
// path for rows longer than 32 * kSelectReg. The attended list is [c, then the
// selected blocks]: ascending when sel_out is requested, else in selection order.
template <int KREG>
__global__ void __launch_bounds__(32) decode_select_kernel(const Params p) {
  __shared__ __align__(16) uint32_t scratch[256];
  const int lane = threadIdx.x;
  const int bg = blockIdx.x;
  griddep_launch_dependents();   // the attention kernel may start its prologue
  const float* srow = p.s + (long long)bg * p.NBmax;
  float sv[KREG > 0 ? KREG : 1];
#pragma unroll
  for (int i = 0; i < KREG; ++i) sv[i] = (lane + 32 * i < p.NBmax) ? __ldg(srow + lane + 32 * i) : 0.f;
  const int b = bg / p.Hkv;
  const int L = p.seqlen[b];
  int32_t* att = p.att + (long long)bg * p.K;
  if (lane == 0) p.tickets[bg] = 0;   // the fp32 attention kernel counts finished blocks here
  if (lane == 0 && bg == 0) *p.work = 0;
  if (L < 1 || L > p.Lmax) {   // a sequence length outside the cache: nothing attended
    if (lane == 0) set_status(p.status, SAS_DEV_ERR_BOUNDS);
    for (int k = lane; k < p.K; k += 32) att[k] = -1;
    return;
  }
  const int c = (L - 1) / kBlock;
  const int H = p.K - 1;
  int32_t* so = p.sel_out ? p.sel_out + (long long)bg * H : nullptr;
  const int mode = (min(c, H) == 0) ? 0 : (c <= H ? 1 : 2);
  if (lane == 0) att[0] = c;
  int pos = -1;
  if constexpr (KREG > 0) {
    if (mode == 2 && H <= 32) {
      uint32_t keys[KREG];
#pragma unroll
      for (int i = 0; i < KREG; ++i) keys[i] = (lane + 32 * i < c) ? float_key(sv[i]) : 0u;
      uint32_t tk = 0u, asc = 0u, top = 0u;
      int tidx = -1;
      if (pivot_select_keys(keys, c, H, reinterpret_cast<uint2*>(scratch), &tk, &tidx, so ? &asc : nullptr,
                            so ? nullptr : &top)) {
        if (lane < H) {
          att[1 + lane] = (int32_t)(so ? asc : top);
          if (so) so[lane] = (int32_t)asc;
        }
        pos = H;
      }
    }
  }
  if (pos < 0) pos = select_row(srow, c, H, mode, scratch, att, so);
  for (int k = 1 + pos + lane; k < p.K; k += 32) att[k] = -1;
  if (so)
    for (int k = pos + lane; k < H; k += 32) so[k] = -1;
  if (p.apply_log_gate) {
    const float lse = row_lse(srow, c);
    if (lane == 0) p.lse_gate[bg] = lse;
  }
  if (p.page_table) map_pages(p, bg, att);
}

constexpr int kLongWarps = 16;   // warps of the long-row selection CTA

// Rows longer than 32 * kSelectReg blocks, any budget: one CTA of kRadixThreads
// threads per (b, g), the row in registers (block m = t + kRadixThreads * i on
// thread t). First a lower bound of the H-th largest key from the warps' four
// largest thread maxima (64 keys of distinct threads): the lesser of the
// ceil(H/2)-th largest of warps 0-7's and of warps 8-15's, so that at least H
// keys of the row are at or above it (0 when some warp holds fewer than four
// keys, which filters nothing). The keys at or above the
// bound are the candidates. When at most kMaxCand of them remain (the usual
// case), each candidate's rank under (key descending, block ascending) is
// counted directly, and the H best are placed by how many taken blocks precede
// them. Otherwise (many keys tied at the bound) an MSB-first radix select over
// shared-memory histograms of the candidates (digits of 11, 11 and 10 bits) finds
// the H-th largest key and how many keys equal to it are taken (the first ones in
// block order), and a scan of the per-(row, warp) counts of larger and of equal
// keys gives each selected block its rank. Either way the list comes out in
// ascending block order.
constexpr int kRadixThreads = 32 * kLongWarps;
constexpr int kRadixBins = 2048;
static_assert(kRadixBins == 4 * kRadixThreads, "each thread owns four histogram bins");
constexpr int kMaxCand = kRadixThreads;   // candidates ranked by counting (one to four threads each)

template <int KR>
__global__ void __launch_bounds__(kRadixThreads) decode_select_radix_kernel(const Params p) {
  __shared__ uint32_t hist[2][kRadixBins];
  __shared__ uint32_t cnt[KR][kLongWarps];   // (larger << 16 | equal) per (row, warp), then exclusive prefixes
  __shared__ int wsum[kLongWarps];
  __shared__ float red[kLongWarps];
  __shared__ uint32_t wtop[4 * kLongWarps];  // per warp: its four largest thread maxima (bound of the select)
  __shared__ uint2 cand[kMaxCand];           // (key, block) of the keys at or above the bound
  __shared__ int taken_flag[kMaxCand];
  __shared__ uint32_t sh_digit, sh_bound;
  __shared__ int sh_rem, n_cand;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bg = blockIdx.x;
  griddep_launch_dependents();   // the attention kernel may start its prologue
  const float* srow = p.s + (long long)bg * p.NBmax;
  float sv[KR];
#pragma unroll
  for (int i = 0; i < KR; ++i) {
    const int m = tid + kRadixThreads * i;
    sv[i] = (m < p.NBmax) ? __ldg(srow + m) : 0.f;
  }
  if (p.page_table) {
    // The sequence's page-table row toward L2 (its Hkv CTAs take a share each), so
    // that the lookups of the selected blocks at the end are L2 hits.
    const int b0 = bg / p.Hkv, g0 = bg % p.Hkv;
    const int lines = (p.max_pages + 31) / 32;   // 128-byte lines of the row
    const int32_t* row = p.page_table + (long long)b0 * p.max_pages;
    for (int l = g0 + p.Hkv * tid; l < lines; l += p.Hkv * kRadixThreads)
      asm volatile("prefetch.global.L2 [%0];" ::"l"(row + min(32 * l, p.max_pages - 1)));
  }
  const int b = bg / p.Hkv;
  const int L = p.seqlen[b];
  int32_t* att = p.att + (long long)bg * p.K;
  if (tid == 0) {
    p.tickets[bg] = 0;
    if (bg == 0) *p.work = 0;
  }
  if (L < 1 || L > p.Lmax) {   // a sequence length outside the cache: nothing attended
    if (tid == 0) set_status(p.status, SAS_DEV_ERR_BOUNDS);
    for (int k = tid; k < p.K; k += kRadixThreads) att[k] = -1;
    return;
  }
  const int c = (L - 1) / kBlock;
  const int H = p.K - 1;
  int32_t* so = p.sel_out ? p.sel_out + (long long)bg * H : nullptr;
  if (tid == 0) att[0] = c;
  if (p.apply_log_gate) {   // log sum_{m < c} exp(s[m]) over the whole CTA
    float mx = -INFINITY;
#pragma unroll
    for (int i = 0; i < KR; ++i)
      if (tid + kRadixThreads * i < c) mx = fmaxf(mx, sv[i]);
#pragma unroll
    for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if (lane == 0) red[warp] = mx;
    __syncthreads();
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kLongWarps; ++w) M = fmaxf(M, red[w]);
    __syncthreads();
    float sum = 0.f;
#pragma unroll
    for (int i = 0; i < KR; ++i)
      if (tid + kRadixThreads * i < c) sum += expf(sv[i] - M);
#pragma unroll
    for (int o = 16; o; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    if (lane == 0) red[warp] = sum;
    __syncthreads();
    if (tid == 0) {
      float tot = 0.f;
      for (int w = 0; w < kLongWarps; ++w) tot += red[w];
      p.lse_gate[bg] = (c > 0) ? M + logf(tot) : 0.f;
    }
  }
  if (c > H && H > 0) {
    uint32_t keys[KR];
#pragma unroll
    for (int i = 0; i < KR; ++i) keys[i] = (tid + kRadixThreads * i < c) ? float_key(sv[i]) : 0u;
    // Lower bound of the H-th largest key (0, no filtering, when some warp holds too few keys).
    uint32_t tmax = 0u;
#pragma unroll
    for (int i = 0; i < KR; ++i) tmax = max(tmax, keys[i]);
    const uint32_t srt = warp_sort_desc(tmax);   // lane j: the warp's j-th largest thread maximum
    if (lane < 4) wtop[4 * warp + lane] = srt;
    if (tid == 0) n_cand = 0;
    __syncthreads();
    if (warp == 0) {
      // Warps 0-7's and warps 8-15's 32 values, each sorted: the k-th largest of
      // each half has k keys of its half at or above it, so the lesser of the two
      // has 2k >= H keys at or above it.
      const uint32_t ha = warp_sort_desc(wtop[lane]);
      const uint32_t hb = warp_sort_desc(wtop[lane + 32]);
      const int k = (H + 1) / 2;   // 1..32
      const uint32_t bnd = min(__shfl_sync(0xffffffffu, ha, k - 1), __shfl_sync(0xffffffffu, hb, k - 1));
      if (lane == 0) sh_bound = bnd;
    }
    __syncthreads();
    const uint32_t bound = sh_bound;
    // The keys at or above the bound (the Top-H among them) go to a shared list.
#pragma unroll
    for (int i = 0; i < KR; ++i) {
      const int m = tid + kRadixThreads * i;
      if (m < c && keys[i] >= bound) {
        const int slot = atomicAdd(&n_cand, 1);
        if (slot < kMaxCand) cand[slot] = make_uint2(keys[i], (uint32_t)m);
      }
    }
    __syncthreads();
    const int n = n_cand;
    if (n <= kMaxCand) {
      // Few candidates: each one's rank under (key descending, block ascending) by
      // counting (tpc threads per candidate); the H best are taken and placed by how
      // many taken blocks precede them.
      const int tpc = n <= kRadixThreads / 4 ? 4 : (n <= kRadixThreads / 2 ? 2 : 1);
      const int j = tid / tpc, q = tid % tpc;
      const bool mine = j < n;
      const uint2 cj = mine ? cand[j] : make_uint2(0u, 0u);
      const uint64_t vj = ((uint64_t)cj.x << 32) | (uint64_t)(0xFFFFFFFFu - cj.y);
      int r = 0;
      if (mine)
        for (int i = q; i < n; i += tpc) {
          const uint2 ci = cand[i];
          r += (((uint64_t)ci.x << 32) | (uint64_t)(0xFFFFFFFFu - ci.y)) > vj ? 1 : 0;
        }
      for (int o = 1; o < tpc; o <<= 1) r += __shfl_xor_sync(0xffffffffu, r, o);
      const bool taken = mine && r < H;
      if (mine && q == 0) taken_flag[j] = taken ? 1 : 0;
      __syncthreads();
      int pc = 0;
      if (taken)
        for (int i = q; i < n; i += tpc) pc += (taken_flag[i] && cand[i].y < cj.y) ? 1 : 0;
      for (int o = 1; o < tpc; o <<= 1) pc += __shfl_xor_sync(0xffffffffu, pc, o);
      if (taken && q == 0) {
        att[1 + pc] = (int32_t)cj.y;
        if (so) so[pc] = (int32_t)cj.y;
      }
    } else {
      // Many keys at the bound (ties): radix select over the keys at or above it.
      for (int jb = tid; jb < kRadixBins; jb += kRadixThreads) hist[0][jb] = 0u;
      __syncthreads();
      uint32_t prefix = 0u;
      int remaining = H;
#pragma unroll 1
      for (int pass = 0; pass < 3; ++pass) {
        const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
        const uint32_t hi_mask = pass == 0 ? 0u : (pass == 1 ? 0xFFE00000u : 0xFFFFFC00u);
        const uint32_t dmask = pass == 2 ? 0x3FFu : 0x7FFu;
        uint32_t* h = hist[pass & 1];
        if (pass < 2)   // the other histogram, for the next pass (its last reader passed a barrier since)
          for (int jb = tid; jb < kRadixBins; jb += kRadixThreads) hist[(pass + 1) & 1][jb] = 0u;
#pragma unroll
        for (int i = 0; i < KR; ++i)
          if (tid + kRadixThreads * i < c && keys[i] >= bound && (keys[i] & hi_mask) == prefix)
            atomicAdd(&h[(keys[i] >> shift) & dmask], 1u);
        __syncthreads();
        // Thread t owns bins 2047-4t .. 2044-4t (descending); a block-wide exclusive
        // scan of the owned counts finds the bin holding the remaining-th largest key.
        int b4[4];
        int loc = 0;
#pragma unroll
        for (int jb = 0; jb < 4; ++jb) {
          b4[jb] = (int)h[kRadixBins - 1 - 4 * tid - jb];
          loc += b4[jb];
        }
        int incl = loc;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int t = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += t;
        }
        if (lane == 31) wsum[warp] = incl;
        __syncthreads();
        int before = incl - loc;
#pragma unroll
        for (int w = 0; w < kLongWarps; ++w) before += (w < warp) ? wsum[w] : 0;
        if (before < remaining && remaining <= before + loc) {
          int run = before;
#pragma unroll
          for (int jb = 0; jb < 4; ++jb) {
            if (run + b4[jb] >= remaining) {
              sh_digit = (uint32_t)(kRadixBins - 1 - 4 * tid - jb);
              sh_rem = remaining - run;
              break;
            }
            run += b4[jb];
          }
        }
        __syncthreads();
        prefix |= sh_digit << shift;
        remaining = sh_rem;
      }
      const uint32_t tkey = prefix;
      const int take_eq = remaining;
      const uint32_t lt = (1u << lane) - 1u;
#pragma unroll
      for (int i = 0; i < KR; ++i) {
        const bool in = tid + kRadixThreads * i < c;
        const uint32_t bgt = __ballot_sync(0xffffffffu, in && keys[i] > tkey);
        const uint32_t beq = __ballot_sync(0xffffffffu, in && keys[i] == tkey);
        if (lane == 0) cnt[i][warp] = ((uint32_t)__popc(bgt) << 16) | (uint32_t)__popc(beq);
      }
      __syncthreads();
      if (warp == 0) {   // exclusive scan over (row, warp) in row-major order = ascending block order
        constexpr int E = KR * kLongWarps;
        constexpr int PER = (E + 31) / 32;
        uint32_t* flat = &cnt[0][0];
        uint32_t v[PER];
        uint32_t lsum = 0u;
#pragma unroll
        for (int jb = 0; jb < PER; ++jb) {
          const int e = lane * PER + jb;
          v[jb] = (e < E) ? flat[e] : 0u;
          lsum += v[jb];
        }
        uint32_t incl = lsum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += t;
        }
        uint32_t run = incl - lsum;
#pragma unroll
        for (int jb = 0; jb < PER; ++jb) {
          const int e = lane * PER + jb;
          if (e < E) flat[e] = run;
          run += v[jb];
        }
      }
      __syncthreads();
#pragma unroll
      for (int i = 0; i < KR; ++i) {
        const int m = tid + kRadixThreads * i;
        const bool in = m < c;
        const bool gt = in && keys[i] > tkey, eq = in && keys[i] == tkey;
        const uint32_t bgt = __ballot_sync(0xffffffffu, gt);
        const uint32_t beq = __ballot_sync(0xffffffffu, eq);
        const uint32_t base = cnt[i][warp];
        const int gt_before = (int)(base >> 16) + __popc(bgt & lt);
        const int eq_before = (int)(base & 0xFFFFu) + __popc(beq & lt);
        if (gt || (eq && eq_before < take_eq)) {
          const int pos = gt_before + min(eq_before, take_eq);
          att[1 + pos] = m;
          if (so) so[pos] = m;
        }
      }
    }
  } else if (warp == 0) {   // nothing to choose: every historical block (c <= H), or none (H == 0)
    const int n = min(c, H);
    for (int m = lane; m < n; m += 32) {
      att[1 + m] = m;
      if (so) so[m] = m;
    }
    for (int k = 1 + n + lane; k < p.K; k += 32) att[k] = -1;
    if (so)
      for (int k = n + lane; k < H; k += 32) so[k] = -1;
  }
  if (p.page_table) {
    __syncthreads();   // every warp wrote part of the list
    if (warp == 0) map_pages(p, bg, att);
  }
}

// ---------------------------------------------------------------------------- attention

// Eight consecutive features of one K or V row as fp32.
__device__ __forceinline__ void load8(const __nv_bfloat16* src, float (&f)[8]) {
  const uint4 raw = *reinterpret_cast<const uint4*>(src);
  const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    f[2 * e] = __uint_as_float(w[e] << 16);
    f[2 * e + 1] = __uint_as_float(w[e] & 0xffff0000u);
  }
}
__device__ __forceinline__ void load8(const float* src, float (&f)[8]) {
  const float4 a = *reinterpret_cast<const float4*>(src);
  const float4 b = *reinterpret_cast<const float4*>(src + 4);
  f[0] = a.x, f[1] = a.y, f[2] = a.z, f[3] = a.w, f[4] = b.x, f[5] = b.y, f[6] = b.z, f[7] = b.w;
}
__device__ __forceinline__ void load8_global(const __nv_bfloat16* src, float (&f)[8]) {
  const uint4 raw = __ldg(reinterpret_cast<const uint4*>(src));
  const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    f[2 * e] = __uint_as_float(w[e] << 16);
    f[2 * e + 1] = __uint_as_float(w[e] & 0xffff0000u);
  }
}
__device__ __forceinline__ void load8_global(const float* src, float (&f)[8]) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(src));
  const float4 b = __ldg(reinterpret_cast<const float4*>(src + 4));
  f[0] = a.x, f[1] = a.y, f[2] = a.z, f[3] = a.w, f[4] = b.x, f[5] = b.y, f[6] = b.z, f[7] = b.w;
}

// Merges the K partials of (b, g) into o: weight_k = exp(max_k - max), o =
// sum_k weight_k o_k / sum_k weight_k sum_k. Run by the NT threads of the CTA
// that took the last ticket; `sm` holds 3*K*G + G floats of shared memory. Every
// load of a phase is independent of the others, so the phase costs about one
// L2 round trip.
template <typename T, int NT, int BATCH>
__device__ __forceinline__ void merge_partials(const Params& p, int bg, float* sm) {
  const int tid = threadIdx.x;
  const int G = p.G, K = p.K;
  const int b = bg / p.Hkv, g = bg % p.Hkv;
  float2* ml = reinterpret_cast<float2*>(sm);   // [K][G] (max, sum) of every partial
  float* wt = sm + 2 * K * G;                   // [K][G] weights
  float* inv = wt + K * G;                      // [G] 1 / denominator
  auto sync = [] {
    if constexpr (NT > 32)
      __syncthreads();
    else
      __syncwarp();
  };
  const float2* pml = reinterpret_cast<const float2*>(p.part_ml + (long long)bg * K * G * 2);
  for (int i = tid; i < K * G; i += NT) ml[i] = __ldcg(pml + i);
  sync();
  for (int h = tid; h < G; h += NT) {
    float M = -INFINITY;
    for (int kk = 0; kk < K; ++kk) M = fmaxf(M, ml[kk * G + h].x);
    float den = 0.f;
    for (int kk = 0; kk < K; ++kk) {
      const float2 v = ml[kk * G + h];
      const float w = (v.x == -INFINITY) ? 0.f : ex2((v.x - M) * kLog2e);
      wt[kk * G + h] = w;
      den = fmaf(w, v.y, den);
    }
    inv[h] = 1.f / den;
  }
  sync();
  const float4* pob = reinterpret_cast<const float4*>(p.part_o + (long long)bg * K * G * D);
  for (int idx = tid; idx < G * (D / 4); idx += NT) {
    const int h = idx / (D / 4), d4 = idx % (D / 4);
    float4 num = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int k0 = 0; k0 < K; k0 += BATCH) {
      float4 u[BATCH];
#pragma unroll
      for (int kk = 0; kk < BATCH; ++kk)
        if (k0 + kk < K) u[kk] = __ldcg(pob + ((k0 + kk) * G + h) * (D / 4) + d4);
#pragma unroll
      for (int kk = 0; kk < BATCH; ++kk) {
        if (k0 + kk < K) {
          // Empty slots were never written: weight zero, and their bits stay unused.
          const float w = wt[(k0 + kk) * G + h];
          if (w != 0.f) {
            num.x = fmaf(w, u[kk].x, num.x);
            num.y = fmaf(w, u[kk].y, num.y);
            num.z = fmaf(w, u[kk].z, num.z);
            num.w = fmaf(w, u[kk].w, num.w);
          }
        }
      }
    }
    const float s = inv[h];
    const long long oi = ((long long)b * p.Hq + g * G + h) * D + d4 * 4;
    if constexpr (sizeof(T) == 2) {
      __nv_bfloat162* dst = reinterpret_cast<__nv_bfloat162*>(static_cast<__nv_bfloat16*>(p.o) + oi);
      dst[0] = __floats2bfloat162_rn(num.x * s, num.y * s);
      dst[1] = __floats2bfloat162_rn(num.z * s, num.w * s);
    } else {
      *reinterpret_cast<float4*>(static_cast<float*>(p.o) + oi) = make_float4(num.x * s, num.y * s, num.z * s, num.w * s);
    }
  }
}

// Merges each (b, g)'s partials (n_slots apiece) into o: one CTA per (b, g),
// launched as a programmatic dependent of the bf16 attention kernel. S adjacent
// threads share one float4 of o, each folding up to 16 slots (one batch of loads
// in flight), and combine their (max, sum, output) states by shuffles.
template <int S>
__host__ __device__ constexpr int merge_threads() {
  return S >= 4 ? 256 : 128 * S;   // up to 16 float4 + 16 float2 loads in flight per thread
}

template <int S>
__global__ void __launch_bounds__(merge_threads<S>()) decode_merge_kernel(const Params p) {
  constexpr int kGroups = merge_threads<S>() / S;   // float4s of o per pass
  griddep_wait();   // the attention kernel's partials are complete and visible
  const int bg = blockIdx.x;
  const int G = p.G, K = p.n_slots;
  const int per = G * (D / 4);
  const int sg = threadIdx.x % S;
  const int k_begin = 16 * sg, k_end = min(K, 16 * sg + 16);
  const int b = bg / p.Hkv, g = bg % p.Hkv;
  for (int base = 0; base < per; base += kGroups) {   // every lane runs every pass (the shuffles)
    const int idx = base + (int)threadIdx.x / S;
    const bool active = idx < per;
    const int h = idx / (D / 4), d4 = idx % (D / 4);
    float M = -INFINITY, den = 0.f;
    float4 num = make_float4(0.f, 0.f, 0.f, 0.f);
    if (active && k_begin < k_end) {
      const float2* pml = reinterpret_cast<const float2*>(p.part_ml) + (long long)bg * K * G + h;
      const float4* pob = reinterpret_cast<const float4*>(p.part_o) + ((long long)bg * K * G + h) * (D / 4) + d4;
      float2 ml[16];
      float4 u[16];
#pragma unroll
      for (int kk = 0; kk < 16; ++kk) {
        if (k_begin + kk < k_end) {
          ml[kk] = __ldcg(pml + (k_begin + kk) * G);
          u[kk] = __ldcg(pob + (long long)(k_begin + kk) * G * (D / 4));
        } else {
          ml[kk] = make_float2(-INFINITY, 0.f);
        }
      }
#pragma unroll
      for (int kk = 0; kk < 16; ++kk) M = fmaxf(M, ml[kk].x);
      if (M != -INFINITY) {
#pragma unroll
        for (int kk = 0; kk < 16; ++kk) {
          // Empty slots (max -inf) were never written: weight zero, bits unused.
          if (ml[kk].x != -INFINITY) {
            const float w = ex2((ml[kk].x - M) * kLog2e);
            den = fmaf(w, ml[kk].y, den);
            num.x = fmaf(w, u[kk].x, num.x);
            num.y = fmaf(w, u[kk].y, num.y);
            num.z = fmaf(w, u[kk].z, num.z);
            num.w = fmaf(w, u[kk].w, num.w);
          }
        }
      }
    }
#pragma unroll
    for (int o = 1; o < S; o <<= 1) {
      const float Mo = __shfl_xor_sync(0xffffffffu, M, o);
      const float deno = __shfl_xor_sync(0xffffffffu, den, o);
      float4 nu;
      nu.x = __shfl_xor_sync(0xffffffffu, num.x, o);
      nu.y = __shfl_xor_sync(0xffffffffu, num.y, o);
      nu.z = __shfl_xor_sync(0xffffffffu, num.z, o);
      nu.w = __shfl_xor_sync(0xffffffffu, num.w, o);
      const float Mn = fmaxf(M, Mo);
      const float a = (M == -INFINITY) ? 0.f : ex2((M - Mn) * kLog2e);
      const float ao = (Mo == -INFINITY) ? 0.f : ex2((Mo - Mn) * kLog2e);
      den = den * a + deno * ao;
      num.x = num.x * a + nu.x * ao;
      num.y = num.y * a + nu.y * ao;
      num.z = num.z * a + nu.z * ao;
      num.w = num.w * a + nu.w * ao;
      M = Mn;
    }
    if (active && sg == 0) {
      const float sc = 1.f / den;
      __nv_bfloat162* dst = reinterpret_cast<__nv_bfloat162*>(static_cast<__nv_bfloat16*>(p.o) +
                                                              ((long long)b * p.Hq + g * G + h) * D + d4 * 4);
      dst[0] = __floats2bfloat162_rn(num.x * sc, num.y * sc);
      dst[1] = __floats2bfloat162_rn(num.z * sc, num.w * sc);
    }
  }
}

// One CTA per work item (b, g, attended block). Lane layout inside a warp: the
// low 16 lanes and the high 16 lanes each cover one whole key row (16 chunks of
// 8 features), so every shared-memory read of a warp is two adjacent rows.
// Warp w owns keys 16w .. 16w+15.
template <typename T>
__global__ void __launch_bounds__(ATT_THREADS, 4) decode_attn_kernel(const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  constexpr uint32_t ROW = D * sizeof(T);      // bytes of one key row
  constexpr uint32_t BLK = kBlock * ROW;       // one K or V block
  const int G = p.G;
  const T* kb = reinterpret_cast<const T*>(smem);
  const T* vb = reinterpret_cast<const T*>(smem + BLK);
  float* red = reinterpret_cast<float*>(smem);                 // reuses the K block once scores are done
  float* sp = reinterpret_cast<float*>(smem + 2 * BLK);        // [G][64] scores, then probabilities
  float* mlb = sp + G * kBlock;                                // [G][2] block max / sum
  uint64_t* bar = reinterpret_cast<uint64_t*>(mlb + 2 * G + 2);
  int* flag = reinterpret_cast<int*>(bar + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int dc = lane & 15, kp = lane >> 4;
  const int bg = blockIdx.x / p.K, k = blockIdx.x % p.K;
  const int b = bg / p.Hkv, g = bg % p.Hkv;
  const int L = p.seqlen[b];
  if (L < 1 || L > p.Lmax) {   // a sequence length outside the cache
    if (threadIdx.x == 0) set_status(p.status, SAS_DEV_ERR_BOUNDS);
    return;
  }
  const int c = (L - 1) / kBlock;
  const long long cache_row0 = (long long)bg * p.Lmax;

  auto issue = [&](int m, int rows) {
    mbar_expect_tx(bar, 2u * rows * ROW);
    const long long off = (cache_row0 + (long long)m * kBlock) * D;
    bulk_copy_g2s(smem_u32(smem), static_cast<const T*>(p.Kc) + off, rows * ROW, bar);
    bulk_copy_g2s(smem_u32(smem + BLK), static_cast<const T*>(p.Vc) + off, rows * ROW, bar);
  };
  if (tid == 0) {
    mbar_init(bar, 1);
    fence_barrier_init();
    if (k == 0) issue(c, L - c * kBlock);   // the current block does not depend on the selection
  }
  // Everything below may read what the selection kernel wrote.
  griddep_wait();
  const int m = (k == 0) ? c : p.att[(long long)bg * p.K + k];
  if (tid == 0 && k != 0 && m >= 0) issue(m, kBlock);
  __syncthreads();

  float* pm = p.part_ml + ((long long)bg * p.K + k) * G * 2;
  float* po = p.part_o + ((long long)bg * p.K + k) * G * D;
  if (m >= 0) {
    const bool ok = __syncthreads_and(mbar_wait(bar, 0, p.status));
    if (!ok) {
      if (tid == 0) mbar_wait_drain(bar, 0);
      return;
    }
    const int nk = (m == c) ? (L - m * kBlock) : kBlock;   // keys present in this block
    const float bias = (p.apply_log_gate && m != c) ? p.s[(long long)bg * p.NBmax + m] - p.lse_gate[bg] : 0.f;
    const T* qg = static_cast<const T*>(p.q) + ((long long)b * p.Hq + g * G) * D;
    // ---- scores, four heads at a time: each lane holds its 8 features of q and
    // forms 8-feature partial dots for 8 keys; a butterfly over the 16 lanes of a
    // row sums them and leaves each lane two finished scores.
    for (int h0 = 0; h0 < G; h0 += HC) {
      float qv[HC][8];
#pragma unroll
      for (int hh = 0; hh < HC; ++hh) {
        if (h0 + hh < G) {
          load8_global(qg + (h0 + hh) * D + dc * 8, qv[hh]);
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e) qv[hh][e] = 0.f;
        }
      }
      float v[HC * 8];   // v[hh * 8 + i]: head h0+hh, key 16*warp + 2*i + kp
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        float kf[8];
        load8(kb + (warp * 16 + 2 * i + kp) * D + dc * 8, kf);
#pragma unroll
        for (int hh = 0; hh < HC; ++hh) {
          float a = 0.f;
#pragma unroll
          for (int e = 0; e < 8; ++e) a = fmaf(qv[hh][e], kf[e], a);
          v[hh * 8 + i] = a;
        }
      }
#pragma unroll
      for (int t = 0; t < 16; ++t) {
        const bool up = lane & 8;
        const float send = up ? v[t] : v[t + 16];
        const float keep = up ? v[t + 16] : v[t];
        v[t] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
      }
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        const bool up = lane & 4;
        const float send = up ? v[t] : v[t + 8];
        const float keep = up ? v[t + 8] : v[t];
        v[t] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
      }
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const bool up = lane & 2;
        const float send = up ? v[t] : v[t + 4];
        const float keep = up ? v[t + 4] : v[t];
        v[t] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
      }
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        const bool up = lane & 1;
        const float send = up ? v[t] : v[t + 2];
        const float keep = up ? v[t + 2] : v[t];
        v[t] = keep + __shfl_xor_sync(0xffffffffu, send, 1);
      }
      // v[e] is the full score of entry j = 2 * dc + e.
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int j = 2 * dc + e, hh = j >> 3, key = warp * 16 + 2 * (j & 7) + kp;
        if (h0 + hh < G) sp[(h0 + hh) * kBlock + key] = (key < nk) ? v[e] * p.sm_scale + bias : -INFINITY;
      }
    }
    __syncthreads();
    // ---- softmax over the block's keys, one warp per head: probabilities relative
    // to the block's own maximum, plus the block's (max, sum).
    for (int h = warp; h < G; h += ATT_THREADS / 32) {
      const float a0 = sp[h * kBlock + lane], a1 = sp[h * kBlock + 32 + lane];
      float mx = fmaxf(a0, a1);
#pragma unroll
      for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      const float e0 = (mx == -INFINITY) ? 0.f : ex2((a0 - mx) * kLog2e);
      const float e1 = (mx == -INFINITY) ? 0.f : ex2((a1 - mx) * kLog2e);
      sp[h * kBlock + lane] = e0;
      sp[h * kBlock + 32 + lane] = e1;
      float sum = e0 + e1;
#pragma unroll
      for (int o = 16; o; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      if (lane == 0) {
        pm[2 * h] = mx;
        pm[2 * h + 1] = sum;
      }
    }
    __syncthreads();
    // ---- P V, four heads at a time: each lane accumulates its 8 features over the
    // warp's keys; the two half-warps are folded by one butterfly step (each half
    // keeps two heads) and the four warps are summed through shared memory.
    for (int h0 = 0; h0 < G; h0 += HC) {
      float acc[HC * 8];
#pragma unroll
      for (int i = 0; i < HC * 8; ++i) acc[i] = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int key = warp * 16 + 2 * i + kp;
        if (key < nk) {   // rows past the end of the cache hold stale bits
          float vf[8];
          load8(vb + key * D + dc * 8, vf);
#pragma unroll
          for (int hh = 0; hh < HC; ++hh) {
            const float w = (h0 + hh < G) ? sp[(h0 + hh) * kBlock + key] : 0.f;
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[hh * 8 + e] = fmaf(w, vf[e], acc[hh * 8 + e]);
          }
        }
      }
#pragma unroll
      for (int t = 0; t < HC * 4; ++t) {
        const float send = kp ? acc[t] : acc[t + HC * 4];
        const float keep = kp ? acc[t + HC * 4] : acc[t];
        acc[t] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
      }
      // acc[hl * 8 + e]: head h0 + 2 * kp + hl, feature 8 * dc + e, summed over the warp's keys.
      if (h0 > 0) __syncthreads();   // the previous chunk's sums have been read
#pragma unroll
      for (int hl = 0; hl < 2; ++hl) {
        float4* dst = reinterpret_cast<float4*>(red + ((warp * HC) + 2 * kp + hl) * D + dc * 8);
        dst[0] = make_float4(acc[hl * 8 + 0], acc[hl * 8 + 1], acc[hl * 8 + 2], acc[hl * 8 + 3]);
        dst[1] = make_float4(acc[hl * 8 + 4], acc[hl * 8 + 5], acc[hl * 8 + 6], acc[hl * 8 + 7]);
      }
      __syncthreads();
      // HC * D / 4 = 128 float4 outputs, one per thread.
      {
        const int hh = tid / (D / 4), d4 = tid % (D / 4);
        if (h0 + hh < G) {
          float4 s4 = reinterpret_cast<const float4*>(red + hh * D)[d4];
#pragma unroll
          for (int w = 1; w < ATT_THREADS / 32; ++w) {
            const float4 u = reinterpret_cast<const float4*>(red + (w * HC + hh) * D)[d4];
            s4.x += u.x, s4.y += u.y, s4.z += u.z, s4.w += u.w;
          }
          reinterpret_cast<float4*>(po + (h0 + hh) * D)[d4] = s4;
        }
      }
    }
  } else {
    // An empty slot (fewer historical blocks than the budget): weight zero in the merge.
    for (int h = tid; h < G; h += ATT_THREADS) {
      pm[2 * h] = -INFINITY;
      pm[2 * h + 1] = 0.f;
    }
  }
  // ---- ticket: the CTA that completes the last item of (b, g) merges the K partials.
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    const int ticket = atomicAdd(p.tickets + bg, 1);
    *flag = (ticket == p.K - 1);
  }
  __syncthreads();
  if (!*flag) return;
  __threadfence();
  merge_partials<T, ATT_THREADS, 4>(p, bg, reinterpret_cast<float*>(smem));   // the K block is free
}

// ---------------------------------------------------------------------------- attention, bf16 (tensor cores)
// One warp (one CTA) per work item (b, g, attended block). The block's K and V
// rows arrive by TMA as two 64-feature boxes each, in the 128-byte swizzle, so
// that the 8-row fragment reads below hit eight different bank groups. The G <= 16
// heads of the group form the 16 rows of m16n8k16 MMAs (bf16 in, fp32
// accumulate): S = q K^T over 8 key tiles and 8 feature steps, a softmax over the
// block in registers, then O = P V over 4 key steps and 16 feature tiles, with P
// taken straight from the S accumulators (the accumulator layout of S is the
// operand layout of P).
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Byte offset of 16-byte chunk `chunk` (0..15) of key row `row` in a K or V tile:
// two boxes of [64 rows][128 bytes] (features 0-63, 64-127), 128-byte swizzle.
__device__ __forceinline__ uint32_t kv_tile_offset(uint32_t row, uint32_t chunk) {
  return (chunk >> 3) * 8192u + row * 128u + (((chunk & 7u) ^ (row & 7u)) << 4);
}

constexpr uint32_t kMmaTileBytes = 2 * 8192;   // one K or V block (64 x 128 bf16)
constexpr int kDecStages = 3;                  // K/V ring stages per CTA
constexpr int kDecWarps = 4;                   // each owns 16 of a block's 64 keys
constexpr uint32_t kStageBytes = 2 * kMmaTileBytes;

// Shared memory of the fused kernel for G heads per group and budget K.
constexpr int kMaxItemsPerCta = 63;            // bounds the per-CTA item and group lists
struct FusedLayout {
  uint32_t q, zero, att, attz, grp, comb, bar, total;
};
__host__ __device__ inline FusedLayout fused_layout(int G, int K) {
  FusedLayout l;
  l.q = kDecStages * kStageBytes;        // 4 q slots of G rows x 256 bytes
  l.zero = l.q + 4u * G * 256u;          // one zero row (q rows G..15 of the MMA)
  l.att = l.zero + 256u;                 // attended block of each of the CTA's items
  l.attz = l.att + 256u;                 // its plane in a paged cache
  l.grp = l.attz + 256u;                 // per (b, g) of the CTA: sequence length, log-gate LSE
  l.comb = l.grp + 2u * 256u;            // [warps][16 rows] (max, sum)
  l.bar = l.comb + kDecWarps * 16 * 2 * 4;
  l.total = l.bar + 128u;                // full/empty barriers, stage blocks, copies in flight
  return l;
}

// Persistent sparse decode attention for bf16 storage: two 4-warp CTAs per SM,
// launched as a programmatic dependent of decode_select_kernel.
//
// CTA i owns the work items u = (b * Hkv + g) * K + k in [u0, u1), consecutive
// (at most 63), and walks them with a 3-stage ring: TMA copies of the next three
// items' K and V blocks (64 keys x 128 features, 128-byte swizzle) are in flight
// while one item is computed. Warp 0 also produces the copies, with the group's q
// rows alongside the first block of each (b, g). Each warp owns 16 of a block's
// 64 keys. The G <= 16 heads of the group are the 16 rows of m16n8k16 MMAs (bf16
// in, fp32 accumulate): S = q K^T for its keys, then O += P V with P taken straight
// from the S accumulators (their layout is the A operand layout). Each warp keeps
// its own online softmax state over the items of one (b, g) (max, sum and output
// in registers; the output is rescaled only when the running max grows by more
// than 2^8). At the end of such a segment the four warps' states are combined by
// fp32 reductions into one partial. decode_merge_kernel, launched as a programmatic
// dependent, merges every (b, g) once all partials are written.
__global__ void __launch_bounds__(32 * kDecWarps, 2)
    decode_fused_mma_kernel(const Params p, const __grid_constant__ CUtensorMap tmk,
                            const __grid_constant__ CUtensorMap tmv, const __grid_constant__ CUtensorMap tmq,
                            const int U) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, gid = lane >> 2, tig = lane & 3;
  const int G = p.G, K = p.K;
  const FusedLayout lay = fused_layout(G, K);
  uint8_t* qring = smem + lay.q;
  uint8_t* zrow = smem + lay.zero;
  int32_t* att_s = reinterpret_cast<int32_t*>(smem + lay.att);
  int32_t* attz_s = reinterpret_cast<int32_t*>(smem + lay.attz);
  int32_t* grp_L = reinterpret_cast<int32_t*>(smem + lay.grp);
  float* grp_lse = reinterpret_cast<float*>(smem + lay.grp + 256u);
  float* comb = reinterpret_cast<float*>(smem + lay.comb);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + lay.bar);
  uint64_t* empty = full + kDecStages;
  int* stage_m = reinterpret_cast<int*>(empty + kDecStages);
  int* issued = stage_m + kDecStages;   // last item index copied into each stage (-1: none)

  const int n_units = p.B * p.Hkv * K;
  const int u0 = blockIdx.x * U, u1 = min(n_units, u0 + U);
  if (u0 >= u1) return;
  const int bg0 = u0 / K, n_grp = (u1 - 1) / K - bg0 + 1;
  if (tid == 0) {
    for (int s = 0; s < kDecStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kDecWarps);
      issued[s] = -1;
    }
    fence_barrier_init();
  }
  if (warp == 0) reinterpret_cast<uint2*>(zrow)[lane] = make_uint2(0u, 0u);
  for (int j = tid; j < n_grp; j += 32 * kDecWarps) grp_L[j] = p.seqlen[(bg0 + j) / p.Hkv];
  griddep_launch_dependents();   // the merge kernel may be scheduled as CTAs finish
  // Everything below may read what the selection kernel wrote.
  griddep_wait();
  for (int i = tid; i < u1 - u0; i += 32 * kDecWarps) att_s[i] = p.att[u0 + i];
  if (p.page_table)
    for (int i = tid; i < u1 - u0; i += 32 * kDecWarps) attz_s[i] = p.att_z[u0 + i];
  if (p.apply_log_gate)
    for (int j = tid; j < n_grp; j += 32 * kDecWarps) grp_lse[j] = p.lse_gate[bg0 + j];
  __syncthreads();

  // ------------------------------------------------------------ producer (warp 0)
  int pf = u0, pf_bg = -1;
  // Fills stage s with the next item: its K/V block (and the group's q rows when
  // the item is the first of its (b, g) here), or a bare arrival for an empty slot.
  auto produce = [&](int s) {
    if (pf >= u1) return;
    if (lane == 0) {
      const int bg = pf / K;
      const bool newbg = bg != pf_bg;
      const int m = att_s[pf - u0];
      stage_m[s] = m;
      const uint32_t bytes = (m >= 0 ? kStageBytes : 0u) + (newbg ? (uint32_t)G * 256u : 0u);
      if (bytes) {
        fence_proxy_async_smem();
        mbar_expect_tx(&full[s], bytes);
        if (newbg) {
          const int b = bg / p.Hkv, g = bg % p.Hkv;
          tma_load_2d(qring + ((bg - bg0) & 3) * G * 256, &tmq, &full[s], 0, b * p.Hq + g * G);
        }
        if (m >= 0) {
          // Contiguous cache: plane bg, rows m*64..; paged: the block's own plane, rows 0..63.
          const int z = p.page_table ? attz_s[pf - u0] : bg;
          const int y = p.page_table ? 0 : m * kBlock;
          uint8_t* st = smem + s * kStageBytes;
          tma_load_3d(st, &tmk, &full[s], 0, y, z);
          tma_load_3d(st + 8192, &tmk, &full[s], 64, y, z);
          tma_load_3d(st + kMmaTileBytes, &tmv, &full[s], 0, y, z);
          tma_load_3d(st + kMmaTileBytes + 8192, &tmv, &full[s], 64, y, z);
        }
        issued[s] = pf - u0;
      } else {
        mbar_arrive(&full[s]);
      }
      pf_bg = bg;
    }
    ++pf;
    __syncwarp();
  };
  if (warp == 0)
    for (int s = 0; s < kDecStages; ++s) produce(s);

  // ------------------------------------------------------------ consumers (all warps)
  // Per-lane parts of the fragment addresses (128-byte swizzle, row & 7 == lane & 7).
  const int r8 = lane & 7, mi = lane >> 3;
  const uint32_t k_row = (uint32_t)(16 * warp + (mi >> 1) * 8 + r8) * 128u;
  const uint32_t v_row = (uint32_t)(16 * warp + (mi & 1) * 8 + r8) * 128u;
  uint32_t k_x[4], v_x[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    k_x[j] = (uint32_t)(((2 * j + (mi & 1)) ^ r8) << 4);
    v_x[j] = (uint32_t)(((2 * j + (mi >> 1)) ^ r8) << 4);
  }
  const int qrow = r8 + (mi & 1) * 8;   // head row this lane addresses in the A fragments of q

  float run_m0 = -INFINITY, run_m1 = -INFINITY, run_l0 = 0.f, run_l1 = 0.f;   // log2 domain
  float oacc[16][4];
#pragma unroll
  for (int nd = 0; nd < 16; ++nd) oacc[nd][0] = oacc[nd][1] = oacc[nd][2] = oacc[nd][3] = 0.f;
  uint32_t qa[8][4];
  int seg_bg = -1, seg_k0 = 0, seg_k1 = 0, q_bg = -1;
  bool ok = true;

  // End of a segment: the warps' states are combined into the partial of slot k0
  // (zeroed when the segment began) and slots k0+1..k1 are marked empty.
  auto flush = [&](int bg, int k0, int k1) {
    float l0 = run_l0, l1 = run_l1;
#pragma unroll
    for (int o = 1; o <= 2; o <<= 1) {
      l0 += __shfl_xor_sync(0xffffffffu, l0, o);
      l1 += __shfl_xor_sync(0xffffffffu, l1, o);
    }
    if (tig == 0) {
      comb[(warp * 16 + gid) * 2] = run_m0;
      comb[(warp * 16 + gid) * 2 + 1] = l0;
      comb[(warp * 16 + gid + 8) * 2] = run_m1;
      comb[(warp * 16 + gid + 8) * 2 + 1] = l1;
    }
    ok = named_bar_and(1, 32 * kDecWarps, ok);
    if (!ok) return;
    float M0 = -INFINITY, M1 = -INFINITY;
#pragma unroll
    for (int w = 0; w < kDecWarps; ++w) {
      M0 = fmaxf(M0, comb[(w * 16 + gid) * 2]);
      M1 = fmaxf(M1, comb[(w * 16 + gid + 8) * 2]);
    }
    const float sc0 = (run_m0 == -INFINITY) ? 0.f : ex2(run_m0 - M0);
    const float sc1 = (run_m1 == -INFINITY) ? 0.f : ex2(run_m1 - M1);
    float* po = p.part_o + ((long long)bg * K + k0) * G * D;
#pragma unroll
    for (int nd = 0; nd < 16; ++nd) {
      if (gid < G) red_add_v2(po + gid * D + nd * 8 + 2 * tig, oacc[nd][0] * sc0, oacc[nd][1] * sc0);
      if (gid + 8 < G) red_add_v2(po + (gid + 8) * D + nd * 8 + 2 * tig, oacc[nd][2] * sc1, oacc[nd][3] * sc1);
    }
    if (warp == 0) {
      float* pm = p.part_ml + (long long)bg * K * G * 2;
      if (tig == 0) {
        float L0 = 0.f, L1 = 0.f;
#pragma unroll
        for (int w = 0; w < kDecWarps; ++w) {
          const float m0 = comb[(w * 16 + gid) * 2], m1 = comb[(w * 16 + gid + 8) * 2];
          if (m0 != -INFINITY) L0 += comb[(w * 16 + gid) * 2 + 1] * ex2(m0 - M0);
          if (m1 != -INFINITY) L1 += comb[(w * 16 + gid + 8) * 2 + 1] * ex2(m1 - M1);
        }
        if (gid < G) {
          pm[(k0 * G + gid) * 2] = (M0 == -INFINITY) ? -INFINITY : M0 * kLn2;
          pm[(k0 * G + gid) * 2 + 1] = L0;
        }
        if (gid + 8 < G) {
          pm[(k0 * G + gid + 8) * 2] = (M1 == -INFINITY) ? -INFINITY : M1 * kLn2;
          pm[(k0 * G + gid + 8) * 2 + 1] = L1;
        }
      }
      for (int i = lane; i < (k1 - k0) * G; i += 32) {
        const int kk = k0 + 1 + i / G, h = i % G;
        pm[(kk * G + h) * 2] = -INFINITY;
        pm[(kk * G + h) * 2 + 1] = 0.f;
      }
    }
    // comb[] is rewritten by the next segment only after every warp has read it.
    named_bar_sync(2, 32 * kDecWarps);
  };

  for (int n = 0, u = u0; u < u1; ++n, ++u) {
    const int s = n % kDecStages;
    const uint32_t ph = (uint32_t)(n / kDecStages) & 1u;
    const int bg = u / K, k = u % K;
    if (bg != seg_bg) {
      if (seg_bg >= 0) flush(seg_bg, seg_k0, seg_k1);
      seg_bg = bg;
      seg_k0 = k;
      run_m0 = run_m1 = -INFINITY;
      run_l0 = run_l1 = 0.f;
#pragma unroll
      for (int nd = 0; nd < 16; ++nd) oacc[nd][0] = oacc[nd][1] = oacc[nd][2] = oacc[nd][3] = 0.f;
      if (warp == 0 && ok) {   // the segment's partial accumulates here by reductions
        float4* po = reinterpret_cast<float4*>(p.part_o + ((long long)bg * K + k) * G * D);
        for (int i = lane; i < G * (D / 4); i += 32) po[i] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
    seg_k1 = k;
    if (ok) ok = warp_wait(&full[s], ph, p.status);
    int m = ok ? stage_m[s] : -1;
    const int L = grp_L[bg - bg0];
    if (L < 1 || L > p.Lmax) m = -1;   // recorded by the selection kernel
    bool zeroed = false;
    if (m >= 0) {
      const int slot = (bg - bg0) & 3;
      const int c = (L - 1) / kBlock;
      const int nk = (m == c) ? (L - m * kBlock) : kBlock;   // keys present in this block
      const uint32_t st = smem_u32(smem + s * kStageBytes);
      if (q_bg != bg) {   // the group's q rows as A fragments; rows G..15 read the zero row
        const uint32_t qa_addr = (qrow < G) ? smem_u32(qring + slot * G * 256 + qrow * 256) + (mi >> 1) * 16u
                                            : smem_u32(zrow);
        const uint32_t qstep = (qrow < G) ? 32u : 0u;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) ldsm_x4(qa_addr + ks * qstep, qa[ks]);
        q_bg = bg;
      }
      if (nk < 16 * warp + 16) {
        // This warp's rows past the end of the sequence may hold any bits; P is zero
        // there, and zero V rows keep 0 * NaN out of the P V products.
        uint8_t* vs = smem + s * kStageBytes + kMmaTileBytes;
        const int row0 = max(nk, 16 * warp);
        for (int i = lane; i < (16 * warp + 16 - row0) * 16; i += 32) {
          const int row = row0 + i / 16, chunk = i % 16;
          *reinterpret_cast<uint4*>(vs + kv_tile_offset(row, chunk)) = make_uint4(0u, 0u, 0u, 0u);
        }
        __syncwarp();
        zeroed = true;
      }
      // ---- S = q K^T for the warp's 16 keys: sacc[j] = rows gid, gid+8, keys 16w + 8j + 2tig, +1.
      float sacc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        uint32_t r[4];
        ldsm_x4(st + (ks >> 2) * 8192u + k_row + k_x[ks & 3], r);
        mma16816(sacc[0], qa[ks], r[0], r[1]);
        mma16816(sacc[1], qa[ks], r[2], r[3]);
      }
      // ---- online softmax (log2 domain).
      const float bias =
          (p.apply_log_gate && m != c) ? p.s[(long long)bg * p.NBmax + m] - grp_lse[bg - bg0] : 0.f;
      const float sl2 = p.sm_scale * kLog2e, bl2 = bias * kLog2e;
#pragma unroll
      for (int j = 0; j < 2; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) sacc[j][e] = fmaf(sacc[j][e], sl2, bl2);
      if (nk < kBlock) {
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
          for (int e = 0; e < 4; ++e)
            if (16 * warp + 8 * j + 2 * tig + (e & 1) >= nk) sacc[j][e] = -INFINITY;
      }
      float mx0 = fmaxf(fmaxf(sacc[0][0], sacc[0][1]), fmaxf(sacc[1][0], sacc[1][1]));
      float mx1 = fmaxf(fmaxf(sacc[0][2], sacc[0][3]), fmaxf(sacc[1][2], sacc[1][3]));
#pragma unroll
      for (int o = 1; o <= 2; o <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
      }
      if (__any_sync(0xffffffffu, mx0 > run_m0 + 8.f || mx1 > run_m1 + 8.f)) {
        const float nm0 = fmaxf(run_m0, mx0), nm1 = fmaxf(run_m1, mx1);
        const float a0 = (run_m0 == -INFINITY) ? 0.f : ex2(run_m0 - nm0);
        const float a1 = (run_m1 == -INFINITY) ? 0.f : ex2(run_m1 - nm1);
        run_m0 = nm0;
        run_m1 = nm1;
        run_l0 *= a0;
        run_l1 *= a1;
#pragma unroll
        for (int nd = 0; nd < 16; ++nd) {
          oacc[nd][0] *= a0;
          oacc[nd][1] *= a0;
          oacc[nd][2] *= a1;
          oacc[nd][3] *= a1;
        }
      }
      const float sub0 = (run_m0 == -INFINITY) ? 0.f : run_m0, sub1 = (run_m1 == -INFINITY) ? 0.f : run_m1;
      float pv[2][4];
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        pv[j][0] = ex2(sacc[j][0] - sub0);
        pv[j][1] = ex2(sacc[j][1] - sub0);
        pv[j][2] = ex2(sacc[j][2] - sub1);
        pv[j][3] = ex2(sacc[j][3] - sub1);
      }
      run_l0 += (pv[0][0] + pv[0][1]) + (pv[1][0] + pv[1][1]);
      run_l1 += (pv[0][2] + pv[0][3]) + (pv[1][2] + pv[1][3]);
      const uint32_t pa[4] = {pack_bf16(pv[0][0], pv[0][1]), pack_bf16(pv[0][2], pv[0][3]),
                              pack_bf16(pv[1][0], pv[1][1]), pack_bf16(pv[1][2], pv[1][3])};
      // ---- O += P V over the warp's 16 keys: oacc[nd] = rows gid, gid+8, features 8nd + 2tig, +1.
      const uint32_t vst = st + kMmaTileBytes;
#pragma unroll
      for (int np = 0; np < 8; ++np) {
        uint32_t r[4];
        ldsm_x4_t(vst + (np >> 2) * 8192u + v_row + v_x[np & 3], r);
        mma16816(oacc[2 * np], pa, r[0], r[1]);
        mma16816(oacc[2 * np + 1], pa, r[2], r[3]);
      }
    }
    if (zeroed) fence_proxy_async_smem();   // the generic writes come before the stage's next copy
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
    if (warp == 0 && ok && pf < u1) {
      // The next item goes into stage s once every warp has finished with it.
      ok = warp_wait(&empty[s], ph, p.status);
      if (ok) produce(s);
    }
  }
  if (seg_bg >= 0) flush(seg_bg, seg_k0, seg_k1);
  if (!ok && warp == 0 && lane == 0) {
    // Wind down: copies still in flight finish before the CTA exits.
    for (int t = 0; t < kDecStages; ++t)
      if (issued[t] >= 0) mbar_wait_drain(&full[t], (uint32_t)(issued[t] / kDecStages) & 1u);
  }
}

// ---------------------------------------------------------------------------- one CTA per (b, g), bf16
// The decode step in one kernel, for problems with about as many groups as SMs:
// CTA (b, g) selects the group's blocks itself, streams them through an NS-stage
// TMA ring and writes the group's G rows of o. No partials, no merge, and the
// copy of the current block (which needs no selection) starts before the
// selection runs.
//
// The producer warp (the last one) loads the sequence length and the score row
// together, starts the copies of q and of the current block, selects the other
// blocks into the attended list in shared memory (and sel_out), then fills one
// stage per attended block as the stages come free; a stage holding block -1
// ends the list. The compute warps form NSET sets of four. Set j takes the list
// positions n = j (mod NSET), from stages n % NS, so the sets work on different
// blocks at once. In a set each warp owns 16 of a block's 64 keys, computed as
// decode_fused_mma_kernel's warps do, with its own online softmax state in
// registers. After the last block the warps' states go to shared memory (the
// ring's first stages, free by then) and are combined in warp order, so the
// result does not depend on timing.
constexpr uint32_t kGrpWarpOut = 16u * D * 4u;   // one warp's [16 rows][D] fp32 output

template <int NSET>
__host__ __device__ constexpr int group_threads() {
  return 32 * (kDecWarps * NSET + 1);
}

struct GroupLayout {
  uint32_t q, zero, comb, att, scratch, bar, total;
};
__host__ __device__ inline GroupLayout group_layout(int NS, int NSET, int K) {
  GroupLayout l;
  l.q = (uint32_t)NS * kStageBytes;      // q rows of the group: up to 16 x 256 bytes
  l.zero = l.q + 16u * 256u;             // one zero row (MMA rows G..15)
  l.comb = l.zero + 256u;                // [compute warps][16 rows] (max, sum)
  l.att = l.comb + (uint32_t)(kDecWarps * NSET) * 16u * 2u * 4u;   // attended list: [current, selected...]
  l.scratch = l.att + ((uint32_t)K * 4u + 15u) / 16u * 16u;   // 256 words for the selection
  l.bar = l.scratch + 1024u;             // barriers, stage blocks, fills, group info
  l.total = l.bar + 256u;
  return l;
}

template <int NS, int NSET, int KREG>
__global__ void __launch_bounds__(group_threads<NSET>(), NS <= 3 ? 2 : 1)
    decode_group_kernel(const Params p, const __grid_constant__ CUtensorMap tmk,
                        const __grid_constant__ CUtensorMap tmv, const __grid_constant__ CUtensorMap tmq) {
  constexpr int kCw = kDecWarps * NSET;   // compute warps; warp kCw produces
  static_assert(NS % NSET == 0, "every stage belongs to one set");
  static_assert(kCw * kGrpWarpOut <= NS * kStageBytes, "the warps' outputs fit in the ring");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, gid = lane >> 2, tig = lane & 3;
  const int G = p.G, K = p.K;
  const int bg = blockIdx.x, b = bg / p.Hkv, g = bg % p.Hkv;
  const GroupLayout lay = group_layout(NS, NSET, K);
  uint8_t* qs = smem + lay.q;
  uint8_t* zrow = smem + lay.zero;
  float* comb = reinterpret_cast<float*>(smem + lay.comb);
  int32_t* att_s = reinterpret_cast<int32_t*>(smem + lay.att);
  uint32_t* sel_scratch = reinterpret_cast<uint32_t*>(smem + lay.scratch);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + lay.bar);
  uint64_t* empty = full + NS;
  uint64_t* qbar = empty + NS;                         // the q rows (one phase)
  int* stage_m = reinterpret_cast<int*>(qbar + 1);     // block in each stage; -1 ends the list
  int* issued = stage_m + NS;                          // last list position placed in each stage (-1: none)
  int* info = issued + NS;   // sequence length, current block, log-gate LSE (float), q copy issued

  if (tid == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kDecWarps);
      issued[s] = -1;
    }
    mbar_init(qbar, 1);
    info[3] = 0;
    fence_barrier_init();
  }
  if (warp == 0) reinterpret_cast<uint2*>(zrow)[lane] = make_uint2(0u, 0u);
  __syncthreads();

  if (warp == kCw) {
    // ------------------------------------------------------------ producer and selection
    const float* srow = p.s + (long long)bg * p.NBmax;
    float sv[KREG];
#pragma unroll
    for (int i = 0; i < KREG; ++i) sv[i] = (lane + 32 * i < p.NBmax) ? __ldg(srow + lane + 32 * i) : 0.f;
    const int L = p.seqlen[b];
    const bool valid = L >= 1 && L <= p.Lmax;
    const int c = valid ? (L - 1) / kBlock : 0;
    if (lane == 0) {
      info[0] = L;
      info[1] = c;
      if (!valid) {   // a sequence length outside the cache: nothing attended
        set_status(p.status, SAS_DEV_ERR_BOUNDS);
      } else {
        info[3] = 1;
        mbar_expect_tx(qbar, (uint32_t)G * 256u);
        tma_load_2d(qs, &tmq, qbar, 0, b * p.Hq + g * G);
        stage_m[0] = c;
        mbar_expect_tx(&full[0], kStageBytes);
        tma_load_3d(smem, &tmk, &full[0], 0, c * kBlock, bg);
        tma_load_3d(smem + 8192, &tmk, &full[0], 64, c * kBlock, bg);
        tma_load_3d(smem + kMmaTileBytes, &tmv, &full[0], 0, c * kBlock, bg);
        tma_load_3d(smem + kMmaTileBytes + 8192, &tmv, &full[0], 64, c * kBlock, bg);
        issued[0] = 0;
      }
    }
    const int H = K - 1;
    int32_t* so = p.sel_out ? p.sel_out + (long long)bg * H : nullptr;
    int pos = 0;
    if (valid) {
      const int mode = (min(c, H) == 0) ? 0 : (c <= H ? 1 : 2);
      pos = -1;
      if (mode == 2 && H <= 32) {
        uint32_t keys[KREG];
#pragma unroll
        for (int i = 0; i < KREG; ++i) keys[i] = (lane + 32 * i < c) ? float_key(sv[i]) : 0u;
        uint32_t tk = 0u, asc = 0u, top = 0u;
        int tidx = -1;
        if (pivot_select_keys(keys, c, H, reinterpret_cast<uint2*>(sel_scratch), &tk, &tidx, so ? &asc : nullptr,
                              so ? nullptr : &top)) {
          if (lane < H) {
            att_s[1 + lane] = (int32_t)(so ? asc : top);
            if (so) so[lane] = (int32_t)asc;
          }
          pos = H;
        }
      }
      if (pos < 0) pos = select_row(srow, c, H, mode, sel_scratch, att_s, so);
      const float lse = p.apply_log_gate ? row_lse(srow, c) : 0.f;
      if (lane == 0) reinterpret_cast<float*>(info)[2] = lse;
    }
    if (so)
      for (int k = pos + lane; k < H; k += 32) so[k] = -1;
    __syncwarp();   // the list (written by every lane) is visible to lane 0
    bool ok = true;
    // Position n of the list goes to stage n % NS. Positions 0..P-1 hold blocks
    // (position 0, the current block, is already on its way); the next NSET
    // positions are end markers, one for each set.
    const int P = valid ? 1 + pos : 0;
    for (int n = valid ? 1 : 0; ok && n < P + NSET; ++n) {
      const int s = n % NS;
      if (n >= NS) ok = warp_wait(&empty[s], (uint32_t)(n / NS - 1) & 1u, p.status);
      if (!ok) break;
      if (lane == 0) {
        if (n < P) {
          const int m = att_s[n];
          stage_m[s] = m;
          fence_proxy_async_smem();
          mbar_expect_tx(&full[s], kStageBytes);
          uint8_t* st = smem + s * kStageBytes;
          tma_load_3d(st, &tmk, &full[s], 0, m * kBlock, bg);
          tma_load_3d(st + 8192, &tmk, &full[s], 64, m * kBlock, bg);
          tma_load_3d(st + kMmaTileBytes, &tmv, &full[s], 0, m * kBlock, bg);
          tma_load_3d(st + kMmaTileBytes + 8192, &tmv, &full[s], 64, m * kBlock, bg);
        } else {
          stage_m[s] = -1;
          mbar_arrive(&full[s]);
        }
        issued[s] = n;
      }
      __syncwarp();
    }
  } else {
    // ------------------------------------------------------------ compute warps
    const int set = warp / kDecWarps, kw = warp % kDecWarps;   // kw: the warp's 16 keys of a block
    const int r8 = lane & 7, mi = lane >> 3;
    const uint32_t k_row = (uint32_t)(16 * kw + (mi >> 1) * 8 + r8) * 128u;
    const uint32_t v_row = (uint32_t)(16 * kw + (mi & 1) * 8 + r8) * 128u;
    uint32_t k_x[4], v_x[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      k_x[j] = (uint32_t)(((2 * j + (mi & 1)) ^ r8) << 4);
      v_x[j] = (uint32_t)(((2 * j + (mi >> 1)) ^ r8) << 4);
    }
    const int qrow = r8 + (mi & 1) * 8;
    float run_m0 = -INFINITY, run_m1 = -INFINITY, run_l0 = 0.f, run_l1 = 0.f;   // log2 domain
    float oacc[16][4];
#pragma unroll
    for (int nd = 0; nd < 16; ++nd) oacc[nd][0] = oacc[nd][1] = oacc[nd][2] = oacc[nd][3] = 0.f;
    uint32_t qa[8][4];
    int L = 0, c = 0;
    bool have_q = false;
    for (int n = set;; n += NSET) {
      const int s = n % NS;
      if (!warp_wait(&full[s], (uint32_t)(n / NS) & 1u, p.status)) break;
      const int m = stage_m[s];
      if (m < 0) break;
      if (!have_q) {   // the group's length was stored before any block's copy; q has its own barrier
        if (!warp_wait(qbar, 0u, p.status)) break;
        have_q = true;
        L = info[0];
        c = info[1];
        const uint32_t qa_addr = (qrow < G) ? smem_u32(qs + qrow * 256) + (mi >> 1) * 16u : smem_u32(zrow);
        const uint32_t qstep = (qrow < G) ? 32u : 0u;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) ldsm_x4(qa_addr + ks * qstep, qa[ks]);
      }
      const int nk = (m == c) ? (L - m * kBlock) : kBlock;   // keys present in this block
      const uint32_t st = smem_u32(smem + s * kStageBytes);
      bool zeroed = false;
      if (nk < 16 * kw + 16) {
        // Rows past the end of the sequence may hold any bits; P is zero there, and
        // zero V rows keep 0 * NaN out of the P V products.
        uint8_t* vs = smem + s * kStageBytes + kMmaTileBytes;
        const int row0 = max(nk, 16 * kw);
        for (int i = lane; i < (16 * kw + 16 - row0) * 16; i += 32) {
          const int row = row0 + i / 16, chunk = i % 16;
          *reinterpret_cast<uint4*>(vs + kv_tile_offset(row, chunk)) = make_uint4(0u, 0u, 0u, 0u);
        }
        __syncwarp();
        zeroed = true;
      }
      float sacc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        uint32_t r[4];
        ldsm_x4(st + (ks >> 2) * 8192u + k_row + k_x[ks & 3], r);
        mma16816(sacc[0], qa[ks], r[0], r[1]);
        mma16816(sacc[1], qa[ks], r[2], r[3]);
      }
      // The list positions past 0 were filled after the log-gate LSE was stored.
      const float bias =
          (p.apply_log_gate && m != c) ? p.s[(long long)bg * p.NBmax + m] - reinterpret_cast<float*>(info)[2] : 0.f;
      const float sl2 = p.sm_scale * kLog2e, bl2 = bias * kLog2e;
#pragma unroll
      for (int j = 0; j < 2; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) sacc[j][e] = fmaf(sacc[j][e], sl2, bl2);
      if (nk < kBlock) {
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
          for (int e = 0; e < 4; ++e)
            if (16 * kw + 8 * j + 2 * tig + (e & 1) >= nk) sacc[j][e] = -INFINITY;
      }
      float mx0 = fmaxf(fmaxf(sacc[0][0], sacc[0][1]), fmaxf(sacc[1][0], sacc[1][1]));
      float mx1 = fmaxf(fmaxf(sacc[0][2], sacc[0][3]), fmaxf(sacc[1][2], sacc[1][3]));
#pragma unroll
      for (int o = 1; o <= 2; o <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
      }
      if (__any_sync(0xffffffffu, mx0 > run_m0 + 8.f || mx1 > run_m1 + 8.f)) {
        const float nm0 = fmaxf(run_m0, mx0), nm1 = fmaxf(run_m1, mx1);
        const float a0 = (run_m0 == -INFINITY) ? 0.f : ex2(run_m0 - nm0);
        const float a1 = (run_m1 == -INFINITY) ? 0.f : ex2(run_m1 - nm1);
        run_m0 = nm0;
        run_m1 = nm1;
        run_l0 *= a0;
        run_l1 *= a1;
#pragma unroll
        for (int nd = 0; nd < 16; ++nd) {
          oacc[nd][0] *= a0;
          oacc[nd][1] *= a0;
          oacc[nd][2] *= a1;
          oacc[nd][3] *= a1;
        }
      }
      const float sub0 = (run_m0 == -INFINITY) ? 0.f : run_m0, sub1 = (run_m1 == -INFINITY) ? 0.f : run_m1;
      float pv[2][4];
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        pv[j][0] = ex2(sacc[j][0] - sub0);
        pv[j][1] = ex2(sacc[j][1] - sub0);
        pv[j][2] = ex2(sacc[j][2] - sub1);
        pv[j][3] = ex2(sacc[j][3] - sub1);
      }
      run_l0 += (pv[0][0] + pv[0][1]) + (pv[1][0] + pv[1][1]);
      run_l1 += (pv[0][2] + pv[0][3]) + (pv[1][2] + pv[1][3]);
      const uint32_t pa[4] = {pack_bf16(pv[0][0], pv[0][1]), pack_bf16(pv[0][2], pv[0][3]),
                              pack_bf16(pv[1][0], pv[1][1]), pack_bf16(pv[1][2], pv[1][3])};
      const uint32_t vst = st + kMmaTileBytes;
#pragma unroll
      for (int np = 0; np < 8; ++np) {
        uint32_t r[4];
        ldsm_x4_t(vst + (np >> 2) * 8192u + v_row + v_x[np & 3], r);
        mma16816(oacc[2 * np], pa, r[0], r[1]);
        mma16816(oacc[2 * np + 1], pa, r[2], r[3]);
      }
      if (zeroed) fence_proxy_async_smem();   // the generic writes come before the stage's next copy
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }
    // ------------------------------------------------------------ combine the compute warps, write o
    float l0 = run_l0, l1 = run_l1;
#pragma unroll
    for (int o = 1; o <= 2; o <<= 1) {
      l0 += __shfl_xor_sync(0xffffffffu, l0, o);
      l1 += __shfl_xor_sync(0xffffffffu, l1, o);
    }
    named_bar_sync(1, 32 * kCw);   // every compute warp is done with the ring
    float* wout = reinterpret_cast<float*>(smem) + warp * (kGrpWarpOut / 4);
    if (tig == 0) {
      comb[(warp * 16 + gid) * 2] = run_m0;
      comb[(warp * 16 + gid) * 2 + 1] = l0;
      comb[(warp * 16 + gid + 8) * 2] = run_m1;
      comb[(warp * 16 + gid + 8) * 2 + 1] = l1;
    }
#pragma unroll
    for (int nd = 0; nd < 16; ++nd) {
      *reinterpret_cast<float2*>(wout + gid * D + nd * 8 + 2 * tig) = make_float2(oacc[nd][0], oacc[nd][1]);
      *reinterpret_cast<float2*>(wout + (gid + 8) * D + nd * 8 + 2 * tig) = make_float2(oacc[nd][2], oacc[nd][3]);
    }
    named_bar_sync(1, 32 * kCw);
    const float* wall = reinterpret_cast<const float*>(smem);
    for (int i = tid; i < G * (D / 4); i += 32 * kCw) {
      const int h = i / (D / 4), d4 = i % (D / 4);
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < kCw; ++w) M = fmaxf(M, comb[(w * 16 + h) * 2]);
      float den = 0.f;
      float4 num = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int w = 0; w < kCw; ++w) {
        const float mw = comb[(w * 16 + h) * 2];
        if (mw != -INFINITY) {
          const float a = ex2(mw - M);
          den = fmaf(a, comb[(w * 16 + h) * 2 + 1], den);
          const float4 v = *reinterpret_cast<const float4*>(wall + w * (kGrpWarpOut / 4) + h * D + d4 * 4);
          num.x = fmaf(a, v.x, num.x);
          num.y = fmaf(a, v.y, num.y);
          num.z = fmaf(a, v.z, num.z);
          num.w = fmaf(a, v.w, num.w);
        }
      }
      const float sc = 1.f / den;
      __nv_bfloat162* dst = reinterpret_cast<__nv_bfloat162*>(static_cast<__nv_bfloat16*>(p.o) +
                                                              ((long long)b * p.Hq + g * G + h) * D + d4 * 4);
      dst[0] = __floats2bfloat162_rn(num.x * sc, num.y * sc);
      dst[1] = __floats2bfloat162_rn(num.z * sc, num.w * sc);
    }
  }
  __syncthreads();
  if (tid == kCw * 32 && *reinterpret_cast<volatile int32_t*>(p.status) != 0) {
    // A wait gave up, so copies may still be in flight: they finish before the CTA
    // exits. Each stage's last fill (a copy or the end marker) is the phase waited
    // for; every earlier phase of the stage completes before it.
    if (info[3]) mbar_wait_drain(qbar, 0u);
    for (int s = 0; s < NS; ++s)
      if (issued[s] >= 0) mbar_wait_drain(&full[s], (uint32_t)(issued[s] / NS) & 1u);
  }
}

size_t smem_bytes(int dtype, int G) {
  const size_t el = dtype == 1 ? 2 : 4;
  return 2 * kBlock * D * el + ((size_t)G * kBlock + 2 * G + 2) * 4 + 8 + 16 + 128;
}

}  // namespace decode

static size_t a256(size_t x) { return (x + 255) / 256 * 256; }

size_t decode_workspace_bytes(int B, int Hq, int Hkv, int K) {
  const int G = Hq / Hkv;
  const size_t n_bg = (size_t)B * Hkv;
  size_t bytes = 256;                                      // status word
  bytes += a256(n_bg * K * sizeof(int32_t));               // attended lists
  bytes += a256(n_bg * K * sizeof(int32_t));               // their planes in a paged cache
  bytes += a256(n_bg * sizeof(float));                     // log-gate LSE
  bytes += a256((n_bg + 1) * sizeof(int32_t));             // tickets, counter
  bytes += a256(n_bg * K * G * 2 * sizeof(float));         // partial max / sum
  bytes += n_bg * K * G * decode::D * sizeof(float);       // partial outputs
  return bytes;
}

cudaError_t launch_decode(const DecodeProblem& pb, void* ws, cudaStream_t st) {
  using namespace decode;
  const int G = pb.Hq / pb.Hkv;
  const size_t n_bg = (size_t)pb.B * pb.Hkv;
  uint8_t* w = static_cast<uint8_t*>(ws);
  Params prm;
  prm.q = pb.q;
  prm.Kc = pb.Kc;
  prm.Vc = pb.Vc;
  prm.seqlen = pb.seqlen;
  prm.s = pb.s;
  prm.o = pb.o;
  prm.sel_out = pb.sel_out;
  prm.status = reinterpret_cast<int32_t*>(w);
  size_t off = 256;
  prm.att = reinterpret_cast<int32_t*>(w + off);
  off += a256(n_bg * pb.K * sizeof(int32_t));
  prm.att_z = reinterpret_cast<int32_t*>(w + off);
  off += a256(n_bg * pb.K * sizeof(int32_t));
  prm.page_table = pb.page_table;
  prm.max_pages = pb.max_pages;
  prm.num_pages = pb.num_pages;
  prm.lse_gate = reinterpret_cast<float*>(w + off);
  off += a256(n_bg * sizeof(float));
  prm.tickets = reinterpret_cast<int32_t*>(w + off);
  prm.work = prm.tickets + n_bg;
  off += a256((n_bg + 1) * sizeof(int32_t));
  prm.part_ml = reinterpret_cast<float*>(w + off);
  off += a256(n_bg * pb.K * G * 2 * sizeof(float));
  prm.part_o = reinterpret_cast<float*>(w + off);
  prm.B = pb.B;
  prm.Hq = pb.Hq;
  prm.Hkv = pb.Hkv;
  prm.Lmax = pb.Lmax;
  prm.NBmax = pb.NBmax;
  prm.K = pb.K;
  prm.apply_log_gate = pb.apply_log_gate;
  prm.G = G;
  prm.n_slots = pb.K;
  prm.sm_scale = pb.sm_scale;
  cudaError_t e;
  if (pb.dtype == 1 && !pb.page_table && pb.NBmax <= 512) {
    // Contiguous bf16 cache, rows of up to 512 blocks and at least three groups
    // per four SMs: the whole step is decode_group_kernel, one CTA
    // per (b, g) (six ring stages and one CTA per SM up to one group per SM,
    // three stages and two CTAs per SM beyond).
    int dev = 0, sms = 148, smem_max = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&smem_max, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) != cudaSuccess)
      return e;
    const int NS = (long long)n_bg <= sms ? 6 : 3;
    const size_t shm = group_layout(NS, NS == 6 ? 2 : 1, pb.K).total + 1024;
    if (4LL * (long long)n_bg >= 3LL * sms && shm <= (size_t)smem_max) {
      CUtensorMap tk, tv, tq;
      if (!make_tmap_bf16_3d(&tk, pb.Kc, D, (uint64_t)pb.Lmax, (uint64_t)n_bg, kBlock) ||
          !make_tmap_bf16_3d(&tv, pb.Vc, D, (uint64_t)pb.Lmax, (uint64_t)n_bg, kBlock) ||
          !make_tmap_bf16_rows(&tq, pb.q, D, (uint64_t)pb.B * pb.Hq, (uint32_t)G))
        return cudaErrorInvalidValue;
      auto group = [&](auto kernel, int threads) -> cudaError_t {
        cudaError_t r = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)shm);
        if (r != cudaSuccess) return r;
        r = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 (int)cudaSharedmemCarveoutMaxShared);
        if (r != cudaSuccess) return r;
        kernel<<<(unsigned)n_bg, threads, shm, st>>>(prm, tk, tv, tq);
        count_launch();
        return cudaGetLastError();
      };
      if (NS == 6) {   // one CTA per SM: two sets of compute warps
        constexpr int t = group_threads<2>();
        if (pb.NBmax <= 128) return group(decode_group_kernel<6, 2, 4>, t);
        if (pb.NBmax <= 256) return group(decode_group_kernel<6, 2, 8>, t);
        return group(decode_group_kernel<6, 2, 16>, t);
      }
      constexpr int t = group_threads<1>();   // two CTAs per SM: one set each
      if (pb.NBmax <= 128) return group(decode_group_kernel<3, 1, 4>, t);
      if (pb.NBmax <= 256) return group(decode_group_kernel<3, 1, 8>, t);
      return group(decode_group_kernel<3, 1, 16>, t);
    }
  }
  // Selection first (it also clears the counters); the attention kernel follows.
  // Both prefer all of L1 as shared memory, so that attention CTAs can start on
  // an SM while a selection CTA still runs there (a carveout change would have to
  // wait for the SM to drain).
  auto select = [&](auto kernel) -> cudaError_t {
    cudaError_t r = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                                         (int)cudaSharedmemCarveoutMaxShared);
    if (r != cudaSuccess) return r;
    kernel<<<(unsigned)n_bg, 32, 0, st>>>(prm);
    count_launch();
    return cudaGetLastError();
  };
  auto select_long = [&](auto kernel) -> cudaError_t {
    cudaError_t r = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                                         (int)cudaSharedmemCarveoutMaxShared);
    if (r != cudaSuccess) return r;
    kernel<<<(unsigned)n_bg, 32 * kLongWarps, 0, st>>>(prm);
    count_launch();
    return cudaGetLastError();
  };
  // Registers per lane for the score row: the row is loaded before its length is known.
  constexpr int kLongSlice = 32 * kLongWarps;   // blocks per CTA and register per lane
  if (pb.NBmax <= 128)
    e = select(decode_select_kernel<4>);
  else if (pb.NBmax <= 256)
    e = select(decode_select_kernel<8>);
  else if (pb.NBmax <= 512)
    e = select(decode_select_kernel<16>);
  else if (pb.NBmax <= 32 * kSelectReg)
    e = select(decode_select_kernel<kSelectReg>);
  else if (pb.NBmax <= 4 * kLongSlice)
    e = select_long(decode_select_radix_kernel<4>);
  else if (pb.NBmax <= 8 * kLongSlice)
    e = select_long(decode_select_radix_kernel<8>);
  else if (pb.NBmax <= 16 * kLongSlice)
    e = select_long(decode_select_radix_kernel<16>);
  else if (pb.NBmax <= 32 * kLongSlice)
    e = select_long(decode_select_radix_kernel<32>);
  else
    e = select(decode_select_kernel<0>);
  if (e != cudaSuccess) return e;
  if (pb.dtype == 1) {
    CUtensorMap tk, tv, tq;
    // Contiguous cache: planes (b, g) of Lmax rows; paged: planes (page, g) of one block.
    const uint64_t rows = pb.page_table ? (uint64_t)kBlock : (uint64_t)pb.Lmax;
    const uint64_t planes = pb.page_table ? (uint64_t)pb.num_pages * pb.Hkv : (uint64_t)n_bg;
    if (!make_tmap_bf16_3d(&tk, pb.Kc, D, rows, planes, kBlock) ||
        !make_tmap_bf16_3d(&tv, pb.Vc, D, rows, planes, kBlock) ||
        !make_tmap_bf16_rows(&tq, pb.q, D, (uint64_t)pb.B * pb.Hq, (uint32_t)G))
      return cudaErrorInvalidValue;
    int dev = 0, sms = 148;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    const long long n_units = (long long)n_bg * pb.K;
    const int per_cta = (int)std::min<long long>(kMaxItemsPerCta, (n_units + 2LL * sms - 1) / (2LL * sms));
    const unsigned grid = (unsigned)((n_units + per_cta - 1) / per_cta);
    const size_t shm = fused_layout(G, pb.K).total + 1024;
    if ((e = cudaFuncSetAttribute(decode_fused_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)shm)) !=
        cudaSuccess)
      return e;
    // All of the unified L1 / shared memory as shared memory: two CTAs (six ring
    // stages of K/V blocks in flight) per SM.
    if ((e = cudaFuncSetAttribute(decode_fused_mma_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                                  (int)cudaSharedmemCarveoutMaxShared)) != cudaSuccess)
      return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(32 * kDecWarps);
    cfg.dynamicSmemBytes = shm;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, decode_fused_mma_kernel, prm, tk, tv, tq, per_cta);
    if (e != cudaSuccess) return e;
    count_launch();
    // The merge of every (b, g), as a programmatic dependent of the attention kernel;
    // S threads per float4 of o, each over at most 16 of the K slots.
    cfg.gridDim = dim3((unsigned)n_bg);
    cfg.dynamicSmemBytes = 0;
    if (pb.K <= 16) {
      cfg.blockDim = dim3(merge_threads<1>());
      e = cudaLaunchKernelEx(&cfg, decode_merge_kernel<1>, prm);
    } else if (pb.K <= 32) {
      cfg.blockDim = dim3(merge_threads<2>());
      e = cudaLaunchKernelEx(&cfg, decode_merge_kernel<2>, prm);
    } else {
      cfg.blockDim = dim3(merge_threads<4>());
      e = cudaLaunchKernelEx(&cfg, decode_merge_kernel<4>, prm);
    }
    if (e != cudaSuccess) return e;
    count_launch();
    return cudaGetLastError();
  }
  const size_t shm = smem_bytes(pb.dtype, G);
  if ((e = cudaFuncSetAttribute(decode_attn_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)shm)) !=
      cudaSuccess)
    return e;
  decode_attn_kernel<float><<<(unsigned)(n_bg * pb.K), ATT_THREADS, shm, st>>>(prm);
  count_launch();
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Allocation-free variant of the decode step.
//
// Its scratch (status word, attended lists, tickets, partials) lives in one
// file-scope device array instead of a caller workspace. Every GPU that loads
// the library keeps this array until the process exits, and every call on a
// device shares it, so calls that overlap on the GPU race on it.
// ---------------------------------------------------------------------------
namespace decode_static {

constexpr size_t kScratchBytes = 8u << 20;   // 8 MiB
static __device__ __align__(256) uint8_t g_decode_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
// Per device: the context the address was looked up in (its process-unique id)
// and the address. A device reset or a released and re-created primary context
// reloads the module, so the array may move: a call from a context with another
// id looks the address up again.
struct ScratchSlot {
  unsigned long long ctx_id;
  void* addr;
};
static ScratchSlot g_scratch[kMaxDevices] = {};
static std::mutex g_scratch_mutex;

// Id of the calling thread's current context (driver entry points resolved once).
static cudaError_t current_context_id(unsigned long long* id) {
  static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
  });
  if (!get_current || !get_id) return cudaErrorNotSupported;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return cudaErrorDeviceUninitialized;
  return get_id(ctx, id) == CUDA_SUCCESS ? cudaSuccess : cudaErrorDeviceUninitialized;
}

// Device address of g_decode_scratch in the current device's context, looked up
// once per context. The host-side name is only a stand-in: the kernels must be
// given this address, never &g_decode_scratch.
static cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  unsigned long long id = 0;
  if (current_context_id(&id) != cudaSuccess) {
    // No current context yet on this thread: cudaSetDevice makes the device's
    // primary context current (it allocates nothing).
    if ((e = cudaSetDevice(dev)) != cudaSuccess) return e;
    if ((e = current_context_id(&id)) != cudaSuccess) return e;
  }
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (g_scratch[dev].addr == nullptr || g_scratch[dev].ctx_id != id) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess) return e;
    g_scratch[dev] = ScratchSlot{id, p};
  }
  *out = g_scratch[dev].addr;
  return cudaSuccess;
}

}  // namespace decode_static

size_t decode_static_scratch_limit() { return decode_static::kScratchBytes; }

cudaError_t launch_decode_static(const DecodeProblem& pb, cudaStream_t st) {
  void* ws = nullptr;
  cudaError_t e = decode_static::scratch_address(&ws);
  if (e != cudaSuccess) return e;
  // The status word starts clear on every call (the select kernel clears the tickets).
  e = cudaMemsetAsync(ws, 0, sizeof(int32_t), st);
  if (e != cudaSuccess) return e;
  return launch_decode(pb, ws, st);
}

cudaError_t decode_static_status(cudaStream_t st, int32_t* out) {
  void* ws = nullptr;
  cudaError_t e = decode_static::scratch_address(&ws);
  if (e != cudaSuccess) return e;
  if ((e = cudaStreamSynchronize(st)) != cudaSuccess) return e;
  return cudaMemcpy(out, ws, sizeof(int32_t), cudaMemcpyDeviceToHost);
}

}  // namespace sas
