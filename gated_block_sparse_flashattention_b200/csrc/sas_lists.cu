// Per-block row lists of the KV-block-outer attention kernels.
//
// The selection of the SAS paper (arXiv 2609.13141, §4.3 "Kernel Design",
// Appendix E) is per query row: position t attends its own block and the
// Top-(K-1) historical blocks m < c_t whose log gate passes the row's threshold
// (logG > tau, or logG == tau and m <= tau_idx). The forward and backward
// kernels run KV-block outer: the CTA of block j of (b, g) visits exactly the
// positions that attend j. This pre-pass turns the thresholds into, per
// (b, g, block), the list of positions that selected the block (the block's own
// 64 positions are implicit), and gives every (position, selected block) pair
// its slot: 1 + the block's rank among the row's selected blocks in ascending
// block order (slot 0 is the row's own block). Rows never hold more than K-1
// selected blocks; a threshold that keeps more has its extra pairs dropped and
// is reported as a device-side bounds error.
//
// The pairs come from thresholding the gates, or, when the caller passes the
// selection's sorted index list (sel), from that list, which is 4*(K-1) bytes
// per row instead of the row's gates.
//
// Three kernels: per-block counts (also kept per chunk of 256 positions), their
// offsets and each chunk's first entry in every list (scans per (b, g)), and the
// lists, placed in one more pass over the rows. A list entry packs the position
// (bits 0-17) and the slot (bits 18-30).
#include <algorithm>

#include "sas_common.cuh"
#include "sas_kernels.h"

namespace sas {
namespace lists {

// Rows per CTA of the count and fill kernels: each CTA aggregates its chunk's
// pairs per block in shared memory and touches the global counters once per
// (chunk, block), so the global atomics do not pile up on a few thousand counters.
constexpr int kChunkRows = 256;

// Calls f(t, m, rank) for every selected historical block m of every position t
// of the chunk (rank: the number of selected blocks of row t below m), and
// done(t, n) once per row with its number of selected blocks. One warp per group
// of 4 positions, blocks strided over the lanes 128 at a time: the loads of the
// 4 rows' 128-block spans are issued together, so a warp pays one round trip per
// group and pass instead of one per row and 32 blocks.
template <typename F, typename Done>
__device__ __forceinline__ void for_each_pair(const float* __restrict__ logG, const float* __restrict__ lse,
                                              const float* __restrict__ tau, const int32_t* __restrict__ tau_idx,
                                              long long bg, int t0, int T, int NB, F&& f, Done&& done) {
  constexpr int R = 4, U = 4;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, n_warps = blockDim.x >> 5;
  const uint32_t below = (1u << lane) - 1u;
  const int t_end = min(T, t0 + kChunkRows);
  for (int tb = t0 + warp * R; tb < t_end; tb += n_warps * R) {
    float tv[R], rl[R];
    int ti[R], c[R], run[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int t = tb + r;
      c[r] = (t < t_end) ? min(t / kBlock, NB) : 0;
      tv[r] = c[r] ? tau[bg * T + t] : 0.f;
      ti[r] = c[r] ? tau_idx[bg * T + t] : 0;
      rl[r] = (c[r] && lse) ? lse[bg * T + t] : 0.f;   // compact gates: log g = s - LSE(s)
      run[r] = 0;
    }
    const int cmax = max(max(c[0], c[1]), max(c[2], c[3]));
    for (int m0 = 0; m0 < cmax; m0 += 32 * U) {
      float x[U][R];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int m = m0 + 32 * u + lane;
#pragma unroll
        for (int r = 0; r < R; ++r) x[u][r] = (m < c[r]) ? logG[(bg * T + tb + r) * (long long)NB + m] - rl[r] : 0.f;
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int m = m0 + 32 * u + lane;
#pragma unroll
        for (int r = 0; r < R; ++r) {
          const bool s = m < c[r] && (x[u][r] > tv[r] || (x[u][r] == tv[r] && m <= ti[r]));
          const uint32_t bal = __ballot_sync(0xffffffffu, s);
          if (s) f(tb + r, m, run[r] + __popc(bal & below));
          run[r] += __popc(bal);
        }
      }
    }
#pragma unroll
    for (int r = 0; r < R; ++r)
      if (lane == r && tb + r < t_end) done(tb + r, run[r]);
  }
}

// The same pairs from the selection's index list: sel[b, g, t, k] (k < H) holds
// row t's selected blocks in ascending order, -1 after the last one, so the
// rank of an entry is its index. This reads 4*H bytes per row instead of the
// row's c_t gates. An entry that is not a historical block of its row (m >= c_t)
// is skipped and reported as a bounds error. One warp per group of 4 rows, the
// rows' loads issued together.
template <typename F, typename Done>
__device__ __forceinline__ void for_each_pair_sel(const int32_t* __restrict__ sel, int H, long long bg, int t0, int T,
                                                  int NB, int32_t* status, F&& f, Done&& done) {
  constexpr int R = 4;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, n_warps = blockDim.x >> 5;
  const int t_end = min(T, t0 + kChunkRows);
  for (int tb = t0 + warp * R; tb < t_end; tb += n_warps * R) {
    int n[R];
#pragma unroll
    for (int r = 0; r < R; ++r) n[r] = 0;
    for (int k0 = 0; k0 < H; k0 += 32) {
      const int k = k0 + lane;
      int m[R];
#pragma unroll
      for (int r = 0; r < R; ++r)
        m[r] = (k < H && tb + r < t_end) ? sel[(bg * T + tb + r) * (long long)H + k] : -1;
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const int c = min((tb + r) / kBlock, NB);
        const bool bad = m[r] >= c;
        if (bad) set_status(status, SAS_DEV_ERR_BOUNDS);
        const bool take = m[r] >= 0 && !bad;
        if (take) f(tb + r, m[r], k);
        n[r] += __popc(__ballot_sync(0xffffffffu, take));
      }
    }
#pragma unroll
    for (int r = 0; r < R; ++r)
      if (lane == r && tb + r < t_end) done(tb + r, n[r]);
  }
}

// Count, per (b, g, block), the positions whose selection contains the block
// (pairs beyond the row's K-1 slots excluded), and keep each chunk's counts
// ccnt[b, g, chunk, block] for the fill. The pairs come from the selection's
// index list when sel is set, else from thresholding the gates. Grid: (chunks of
// T, B * Hkv); dynamic shared memory: NB ints.
__global__ void __launch_bounds__(256) count_kernel(const float* __restrict__ logG, const float* __restrict__ lse,
                                                    const float* __restrict__ tau,
                                                    const int32_t* __restrict__ tau_idx,
                                                    const int32_t* __restrict__ sel, int32_t* __restrict__ cnt,
                                                    int32_t* __restrict__ ccnt, int32_t* status, int T, int NB,
                                                    int H) {
  extern __shared__ int32_t hist[];
  const long long bg = blockIdx.y;
  const int t0 = blockIdx.x * kChunkRows;
  for (int m = threadIdx.x; m < NB; m += blockDim.x) hist[m] = 0;
  __syncthreads();
  bool over = false;
  auto add = [&](int, int m, int rank) {
    if (rank < H) atomicAdd(hist + m, 1);
  };
  auto row_done = [&](int, int n) { over |= n > H; };
  if (sel)
    for_each_pair_sel(sel, H, bg, t0, T, NB, status, add, row_done);
  else
    for_each_pair(logG, lse, tau, tau_idx, bg, t0, T, NB, add, row_done);
  if (over) set_status(status, SAS_DEV_ERR_BOUNDS);
  __syncthreads();
  int32_t* cc = ccnt + (bg * gridDim.x + blockIdx.x) * NB;
  for (int m = threadIdx.x; m < NB; m += blockDim.x) {
    const int v = hist[m];
    cc[m] = v;
    if (v) atomicAdd(cnt + bg * NB + m, v);
  }
}

// Offsets: each (b, g) owns a region of T * min(H, NB) entries; off = region +
// prefix of the block counts. Then each chunk's first entry in each block's list:
// ccnt[b, g, chunk, m] becomes the prefix of the earlier chunks' counts (chunk
// order = position order, so every list is ordered by chunk).
__global__ void __launch_bounds__(1024) offsets_kernel(const int32_t* __restrict__ cnt, int32_t* __restrict__ off,
                                                       int32_t* __restrict__ ccnt, int32_t* __restrict__ cap,
                                                       int32_t* __restrict__ total, int32_t* status, int NB,
                                                       int n_chunks, long long region) {
  __shared__ int32_t warp_sums[32];
  const long long bg = blockIdx.x;
  int base = 0;
  for (int j0 = 0; j0 < NB; j0 += 1024) {
    const int j = j0 + threadIdx.x;
    const int v = j < NB ? cnt[bg * NB + j] : 0;
    int incl = v;
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += u;
    }
    if (lane == 31) warp_sums[w] = incl;
    __syncthreads();
    if (w == 0) {
      int ws = warp_sums[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, ws, o);
        if (lane >= o) ws += u;
      }
      warp_sums[lane] = ws;
    }
    __syncthreads();
    const int excl = incl - v + (w > 0 ? warp_sums[w - 1] : 0);
    if (j < NB) {
      // With at most H pairs per row the lists fit their region; the cut is a
      // guard that keeps every write inside it whatever the counts say.
      const long long start = base + excl;
      const long long room = region - start;
      off[bg * NB + j] = (int32_t)(bg * region + (start < region ? start : region));
      cap[bg * NB + j] = (int32_t)(room <= 0 ? 0 : (room < v ? room : v));
      if (room < v) set_status(status, SAS_DEV_ERR_BOUNDS);
      int32_t* cc = ccnt + bg * n_chunks * NB + j;
      int run = 0;
      for (int c0 = 0; c0 < n_chunks; c0 += 16) {   // 16 loads in flight, then their prefix
        int x[16];
#pragma unroll
        for (int u = 0; u < 16; ++u) x[u] = (c0 + u < n_chunks) ? cc[(long long)(c0 + u) * NB] : 0;
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          if (c0 + u < n_chunks) cc[(long long)(c0 + u) * NB] = run;
          run += x[u];
        }
      }
    }
    base += warp_sums[31];
    __syncthreads();
  }
  if (threadIdx.x == 0) total[bg] = (int32_t)(base < region ? base : region);   // entries in use
}

// Writes the lists: each chunk places its pairs of block m from its own first
// entry on (offsets_kernel), a shared-memory counter per block giving the next
// free one. Also writes nsel[t], the number of selected blocks of each row
// (capped at H), when nsel is not null. Grid: (chunks of T, B * Hkv); dynamic
// shared memory: 2 * NB ints.
__global__ void __launch_bounds__(256) fill_kernel(const float* __restrict__ logG, const float* __restrict__ lse,
                                                   const float* __restrict__ tau,
                                                   const int32_t* __restrict__ tau_idx,
                                                   const int32_t* __restrict__ sel, int32_t* status,
                                                   const int32_t* __restrict__ off, const int32_t* __restrict__ cap,
                                                   const int32_t* __restrict__ cbase, int32_t* __restrict__ list,
                                                   int32_t* __restrict__ nsel, int T, int NB, int H) {
  extern __shared__ int32_t sm[];
  int32_t* lcnt = sm;        // entries placed so far per block
  int32_t* lbase = sm + NB;  // the chunk's first entry in each block's list
  const long long bg = blockIdx.y;
  const int t0 = blockIdx.x * kChunkRows;
  const int32_t* cb = cbase + (bg * gridDim.x + blockIdx.x) * NB;
  for (int m = threadIdx.x; m < NB; m += blockDim.x) {
    lcnt[m] = 0;
    lbase[m] = cb[m];
  }
  __syncthreads();
  auto place = [&](int t, int m, int rank) {
    if (rank >= H) return;
    const int at = lbase[m] + atomicAdd(lcnt + m, 1);
    if (at < cap[bg * NB + m]) list[off[bg * NB + m] + at] = t | ((rank + 1) << kEntrySlotShift);
  };
  auto row_done = [&](int t, int n) {
    if (nsel) nsel[bg * T + t] = min(n, H);
  };
  if (sel)
    for_each_pair_sel(sel, H, bg, t0, T, NB, status, place, row_done);
  else
    for_each_pair(logG, lse, tau, tau_idx, bg, t0, T, NB, place, row_done);
}

}  // namespace lists

static int n_chunks_of(int T) { return (T + lists::kChunkRows - 1) / lists::kChunkRows; }

size_t block_lists_bytes(long long nbg, int T, int NB, int K) {
  const long long region = (long long)T * std::max(1, std::min(K - 1, NB));
  auto a256 = [](size_t x) { return (x + 255) / 256 * 256; };
  return 3 * a256((size_t)nbg * NB * sizeof(int32_t))                 // counts, offsets, caps
         + a256((size_t)nbg * n_chunks_of(T) * NB * sizeof(int32_t))   // per-chunk counts, then bases
         + a256((size_t)nbg * region * sizeof(int32_t))                // entries
         + a256((size_t)nbg * T * sizeof(int32_t))                     // selected blocks per row
         + a256((size_t)nbg * sizeof(int32_t));                        // entries in use per (b, g)
}

BlockLists carve_block_lists(uint8_t* scratch, long long nbg, int T, int NB, int K) {
  auto a256 = [](size_t x) { return (x + 255) / 256 * 256; };
  BlockLists L;
  L.region = (long long)T * std::max(1, std::min(K - 1, NB));
  size_t o = 0;
  L.cnt = reinterpret_cast<int32_t*>(scratch + o);
  o += a256((size_t)nbg * NB * sizeof(int32_t));
  L.off = reinterpret_cast<int32_t*>(scratch + o);
  o += a256((size_t)nbg * NB * sizeof(int32_t));
  L.cap = reinterpret_cast<int32_t*>(scratch + o);
  o += a256((size_t)nbg * NB * sizeof(int32_t));
  L.ccnt = reinterpret_cast<int32_t*>(scratch + o);
  o += a256((size_t)nbg * n_chunks_of(T) * NB * sizeof(int32_t));
  L.list = reinterpret_cast<int32_t*>(scratch + o);
  o += a256((size_t)nbg * L.region * sizeof(int32_t));
  L.nsel = reinterpret_cast<int32_t*>(scratch + o);
  o += a256((size_t)nbg * T * sizeof(int32_t));
  L.total = reinterpret_cast<int32_t*>(scratch + o);
  return L;
}

cudaError_t launch_block_lists(const float* logG, const float* gate_lse, const float* tau, const int32_t* tau_idx,
                               const int32_t* sel, const BlockLists& L,
                               long long nbg, int T, int NB, int K, bool want_nsel, int32_t* status,
                               cudaStream_t st) {
  using namespace lists;
  const int H = std::max(0, K - 1);
  const int n_chunks = n_chunks_of(T);
  cudaError_t e = cudaMemsetAsync(L.cnt, 0, (size_t)nbg * NB * sizeof(int32_t), st);
  if (e != cudaSuccess) return e;
  const dim3 chunks((unsigned)n_chunks, (unsigned)nbg);
  count_kernel<<<chunks, 256, NB * sizeof(int32_t), st>>>(logG, gate_lse, tau, tau_idx, H > 0 ? sel : nullptr,
                                                           L.cnt, L.ccnt, status, T, NB, H);
  count_launch();
  offsets_kernel<<<(unsigned)nbg, 1024, 0, st>>>(L.cnt, L.off, L.ccnt, L.cap, L.total, status, NB, n_chunks,
                                                   L.region);
  count_launch();
  fill_kernel<<<chunks, 256, 2 * NB * sizeof(int32_t), st>>>(logG, gate_lse, tau, tau_idx, H > 0 ? sel : nullptr,
                                                              status, L.off, L.cap, L.ccnt, L.list,
                                                              want_nsel ? L.nsel : nullptr, T, NB, H);
  count_launch();
  return cudaGetLastError();
}

}  // namespace sas
