// SAS sparse decode step (memory-bound).
//
// SAS paper (arXiv 2609.13141) §4.3 Algorithm 2 (Top-K on the selector scores,
// then ungated attention over the current block and the selected blocks) and
// §5.1 "Inference implementation" (per-KV-group selection, GQA, gathering only
// the selected KV blocks).
//
// Two kernels:
//   decode_select_kernel  one warp per (b, g): radix select of the Top-(K-1)
//                         historical blocks on the score row; the attended
//                         list [c, selected blocks ascending] goes to the workspace.
//   decode_attn_kernel    persistent, two CTAs per SM. Work items are (b, g,
//                         attended block); warp 0 streams each item's K and V
//                         block (64 keys x 128 features, two 16 KiB bulk async
//                         copies) into a 3-stage ring, 8 compute warps score the
//                         G heads against it, run a softmax over the block and
//                         accumulate P V, and write an fp32 partial (row max,
//                         row sum, unnormalised output). The CTA that finishes the
//                         last item of a (b, g) (atomic ticket) merges its partials.
#include <algorithm>
#include <mutex>

#include "sas_common.cuh"
#include "sas_kernels.h"

namespace sas {
namespace decode {

constexpr int D = 128;
constexpr int NS = 3;                    // K/V ring stages
constexpr int COMPUTE_WARPS = 8;
constexpr int THREADS = 32 * (1 + COMPUTE_WARPS);

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
  int32_t* tickets;    // [B*Hkv]
  float* part_ml;      // [B*Hkv][K][G][2]
  float* part_o;       // [B*Hkv][K][G][D]
  int B, Hq, Hkv, Lmax, NBmax, K, apply_log_gate, G, n_items;
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

// ---------------------------------------------------------------------------- selection
__global__ void __launch_bounds__(256) decode_select_kernel(const Params p) {
  __shared__ uint32_t hist_all[8][256];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int bg = blockIdx.x * 8 + wid;
  if (bg >= p.B * p.Hkv) return;
  const int b = bg / p.Hkv;
  const int L = p.seqlen[b];
  const int c = (L - 1) / kBlock;
  const int H = p.K - 1;
  const float* srow = p.s + (long long)bg * p.NBmax;
  int32_t* att = p.att + (long long)bg * p.K;
  int32_t* so = p.sel_out ? p.sel_out + (long long)bg * H : nullptr;
  // mode 0: nothing selected; 1: every historical block; 2: threshold (tk, tidx).
  const int mode = (min(c, H) == 0) ? 0 : (c <= H ? 1 : 2);
  if (lane == 0) att[0] = c;
  int pos = 0;
  if (c <= 32 * kSelectReg) {
    uint32_t keys[kSelectReg];
    load_row_keys(srow, c, keys);
    uint32_t tk = 0u;
    int tidx = -1;
    if (mode == 2) {
      int take_eq = 0;
      tk = radix_select_keys(keys, c, H, hist_all[wid], &take_eq);
      tidx = tie_index_keys(keys, c, tk, take_eq);
    }
#pragma unroll
    for (int i = 0; i < kSelectReg; ++i) {
      if (mode == 0 || 32 * i >= c) break;
      const int m = lane + 32 * i;
      const bool take = m < c && (mode == 1 || keys[i] > tk || (keys[i] == tk && m <= tidx));
      const uint32_t bal = __ballot_sync(0xffffffffu, take);
      if (take) {
        const int lp = pos + __popc(bal & ((1u << lane) - 1u));
        att[1 + lp] = m;
        if (so) so[lp] = m;
      }
      pos += __popc(bal);
    }
  } else {
    uint32_t tk = 0u;
    int tidx = -1;
    if (mode == 2) {
      int take_eq = 0;
      tk = radix_select_global(srow, c, H, hist_all[wid], &take_eq);
      tidx = tie_index_global(srow, c, tk, take_eq);
    }
    for (int base = 0; mode != 0 && base < c; base += 32) {
      const int m = base + lane;
      bool take = false;
      if (m < c) {
        const uint32_t k = float_key(srow[m]);
        take = mode == 1 || (k > tk) || (k == tk && m <= tidx);
      }
      const uint32_t bal = __ballot_sync(0xffffffffu, take);
      if (take) {
        const int lp = pos + __popc(bal & ((1u << lane) - 1u));
        att[1 + lp] = m;
        if (so) so[lp] = m;
      }
      pos += __popc(bal);
    }
  }
  for (int k = 1 + pos + lane; k < p.K; k += 32) att[k] = -1;
  if (so)
    for (int k = pos + lane; k < H; k += 32) so[k] = -1;
  if (p.apply_log_gate) {
    float mx = -INFINITY;
    for (int m = lane; m < c; m += 32) mx = fmaxf(mx, srow[m]);
#pragma unroll
    for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float sum = 0.f;
    for (int m = lane; m < c; m += 32) sum += expf(srow[m] - mx);
#pragma unroll
    for (int o = 16; o; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    if (lane == 0) p.lse_gate[bg] = (c > 0) ? mx + logf(sum) : 0.f;
  }
}

// ---------------------------------------------------------------------------- attention
template <typename T>
__global__ void __launch_bounds__(THREADS, 2) decode_attn_kernel(const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  constexpr uint32_t BLK = 64 * D * sizeof(T);          // one K or V block
  constexpr int CT = 32 * COMPUTE_WARPS;                // compute threads
  uint8_t* ring = smem;                                 // [NS][K block, V block]
  float* qf = reinterpret_cast<float*>(smem + NS * 2 * BLK);   // [G][D] of the current (b, g)
  float* pr = qf + p.G * D;                                    // [G][64] scores, then probabilities
  float* qsum = pr + p.G * 64;                                 // [4][G][D] partial P V sums
  float* acc_o = qsum + 4 * p.G * D;                           // [G][D] running output of the segment
  float* acc_ml = acc_o + p.G * D;                             // [G][2] running max / sum; [G][2] item max / sum
  float* fac = acc_ml + 4 * p.G;                               // [G][2] rescale factors of one fold
  uint64_t* full = reinterpret_cast<uint64_t*>(fac + 2 * p.G);
  uint64_t* empty = full + NS;
  int* last_flag = reinterpret_cast<int*>(empty + NS);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int per_cta = (p.n_items + gridDim.x - 1) / gridDim.x;
  const int it0 = blockIdx.x * per_cta;
  const int it1 = min(p.n_items, it0 + per_cta);
  const int G = p.G;
  if (tid == 0) {
    for (int i = 0; i < NS; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], COMPUTE_WARPS);
    }
    fence_barrier_init();
  }
  __syncthreads();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int issued = 0;
      for (int it = it0; it < it1; ++it) {
        const int n = it - it0, st = n % NS;
        if (n >= NS && !mbar_wait(&empty[st], ((n / NS) - 1) & 1, p.status)) break;
        const int bg = it / p.K, k = it % p.K;
        const int m = p.att[(long long)bg * p.K + k];
        issued = n + 1;
        if (m < 0) {
          mbar_arrive(&full[st]);   // empty item: nothing to copy
          continue;
        }
        const int rows = min(kBlock, p.Lmax - m * kBlock);
        const long long off = ((long long)bg * p.Lmax + (long long)m * kBlock) * D;
        mbar_expect_tx(&full[st], 2u * rows * D * sizeof(T));
        const uint32_t dst = smem_u32(ring + st * 2 * BLK);
        bulk_copy_g2s(dst, static_cast<const T*>(p.Kc) + off, rows * D * sizeof(T), &full[st]);
        bulk_copy_g2s(dst + BLK, static_cast<const T*>(p.Vc) + off, rows * D * sizeof(T), &full[st]);
      }
      // Copies still in flight finish before the CTA exits.
      for (int n = max(0, issued - NS); n < issued; ++n) mbar_wait_drain(&full[n % NS], (n / NS) & 1);
    }
    return;
  }
  // ------------------------------------------------------------ compute warps
  // Items of one (b, g) that this CTA processes back to back form a segment; the
  // segment keeps a running (max, sum, output) in shared memory (online softmax)
  // and leaves one partial, in the slot of its first item.
  const int ct = tid - 32;
  int cur_bg = -1, seg_k0 = 0;
  for (int it = it0; it < it1; ++it) {
    const int n = it - it0, st = n % NS;
    const int bg = it / p.K, k = it % p.K;
    const int b = bg / p.Hkv, g = bg % p.Hkv;
    const int L = p.seqlen[b];
    const int c = (L - 1) / kBlock;
    const int m = p.att[(long long)bg * p.K + k];
    if (bg != cur_bg) {   // new segment: q of the group's heads (fp32), accumulator reset
      named_bar_sync(1, CT);
      const T* qg = static_cast<const T*>(p.q) + ((long long)b * p.Hq + g * G) * D;
      for (int i = ct; i < G * D; i += CT) {
        qf[i] = to_f<T>(qg[i]);
        acc_o[i] = 0.f;
      }
      for (int h = ct; h < G; h += CT) {
        acc_ml[2 * h] = -INFINITY;
        acc_ml[2 * h + 1] = 0.f;
      }
      named_bar_sync(1, CT);
      cur_bg = bg;
      seg_k0 = k;
    }
    // All compute warps agree on success before going on (they meet at named barriers).
    if (!named_bar_and(2, CT, warp_wait(&full[st], (n / NS) & 1, p.status))) break;
    if (m >= 0) {
      const T* kb = reinterpret_cast<const T*>(ring + st * 2 * BLK);
      const T* vb = reinterpret_cast<const T*>(ring + st * 2 * BLK + BLK);
      const int nk = (m == c) ? (L - m * kBlock) : kBlock;   // keys present in this block
      const float bias = (p.apply_log_gate && m != c) ? p.s[(long long)bg * p.NBmax + m] - p.lse_gate[bg] : 0.f;
      // Scores: thread = (key, quarter of the features), four heads at a time; the
      // four quarters of a key sit in adjacent lanes and are summed by shuffles.
      // Chunks are read in a key-rotated order to spread the shared-memory banks.
      {
        const int quarter = ct & 3, key = ct >> 2;   // 256 threads = 64 keys x 4 quarters
        const T* kr = kb + key * D + quarter * 32;
        float kv[32];   // kv[8*j + e] = element e of chunk (j + key) & 3
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int cc = (j + key) & 3;
          if constexpr (sizeof(T) == 2) {
            const uint4 raw = *reinterpret_cast<const uint4*>(kr + cc * 8);
            const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 f = __bfloat1622float2(h2[e]);
              kv[j * 8 + 2 * e] = f.x;
              kv[j * 8 + 2 * e + 1] = f.y;
            }
          } else {
            const float4 a0 = *reinterpret_cast<const float4*>(kr + cc * 8);
            const float4 a1 = *reinterpret_cast<const float4*>(kr + cc * 8 + 4);
            kv[j * 8 + 0] = a0.x;
            kv[j * 8 + 1] = a0.y;
            kv[j * 8 + 2] = a0.z;
            kv[j * 8 + 3] = a0.w;
            kv[j * 8 + 4] = a1.x;
            kv[j * 8 + 5] = a1.y;
            kv[j * 8 + 6] = a1.z;
            kv[j * 8 + 7] = a1.w;
          }
        }
        for (int h0 = 0; h0 < G; h0 += 4) {
          float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int hh = 0; hh < 4; ++hh) {
            if (h0 + hh < G) {
              const float* qh = qf + (h0 + hh) * D + quarter * 32;
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                const int cc = (j + key) & 3;
                const float4 q0 = *reinterpret_cast<const float4*>(qh + cc * 8);
                const float4 q1 = *reinterpret_cast<const float4*>(qh + cc * 8 + 4);
                acc[hh] = fmaf(q0.x, kv[j * 8 + 0], acc[hh]);
                acc[hh] = fmaf(q0.y, kv[j * 8 + 1], acc[hh]);
                acc[hh] = fmaf(q0.z, kv[j * 8 + 2], acc[hh]);
                acc[hh] = fmaf(q0.w, kv[j * 8 + 3], acc[hh]);
                acc[hh] = fmaf(q1.x, kv[j * 8 + 4], acc[hh]);
                acc[hh] = fmaf(q1.y, kv[j * 8 + 5], acc[hh]);
                acc[hh] = fmaf(q1.z, kv[j * 8 + 6], acc[hh]);
                acc[hh] = fmaf(q1.w, kv[j * 8 + 7], acc[hh]);
              }
            }
          }
#pragma unroll
          for (int hh = 0; hh < 4; ++hh) {
            float a = acc[hh];
            a += __shfl_xor_sync(0xffffffffu, a, 1);
            a += __shfl_xor_sync(0xffffffffu, a, 2);
            if (quarter == 0 && h0 + hh < G) pr[(h0 + hh) * 64 + key] = (key < nk) ? a * p.sm_scale + bias : -INFINITY;
          }
        }
      }
      named_bar_sync(1, CT);
      // Softmax over the block's 64 keys: one warp per head; the item's (max, sum)
      // and the fold factors into the segment accumulator.
      for (int h = ct >> 5; h < G; h += COMPUTE_WARPS) {
        const float a0 = pr[h * 64 + lane], a1 = pr[h * 64 + 32 + lane];
        float mx = fmaxf(a0, a1);
#pragma unroll
        for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        const float e0 = (mx == -INFINITY) ? 0.f : expf(a0 - mx);
        const float e1 = (mx == -INFINITY) ? 0.f : expf(a1 - mx);
        pr[h * 64 + lane] = e0;
        pr[h * 64 + 32 + lane] = e1;
        float sum = e0 + e1;
#pragma unroll
        for (int o = 16; o; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        if (lane == 0) {
          const float m_old = acc_ml[2 * h], l_old = acc_ml[2 * h + 1];
          const float m_new = fmaxf(m_old, mx);
          const float f_old = (m_old == -INFINITY) ? 0.f : expf(m_old - m_new);
          const float f_item = (mx == -INFINITY) ? 0.f : expf(mx - m_new);
          fac[2 * h] = f_old;
          fac[2 * h + 1] = f_item;
          acc_ml[2 * h] = m_new;
          acc_ml[2 * h + 1] = l_old * f_old + sum * f_item;
        }
      }
      named_bar_sync(1, CT);
      // P V: thread = (feature pair, quarter of the keys), features fastest across
      // lanes (conflict-free V reads), four heads at a time; quarters summed in smem.
      {
        const int dp = ct & 63, kq = ct >> 6;
        const int k_lo = kq * 16, k_hi = min(nk, k_lo + 16);
        float2* part = reinterpret_cast<float2*>(qsum);   // [4 quarters][G][64 pairs]
        for (int h0 = 0; h0 < G; h0 += 4) {
          float o0[4] = {0.f, 0.f, 0.f, 0.f}, o1[4] = {0.f, 0.f, 0.f, 0.f};
          for (int key = k_lo; key < k_hi; ++key) {
            float v0, v1;
            if constexpr (sizeof(T) == 2) {
              const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(vb + key * D + 2 * dp));
              v0 = f.x;
              v1 = f.y;
            } else {
              const float2 f = *reinterpret_cast<const float2*>(vb + key * D + 2 * dp);
              v0 = f.x;
              v1 = f.y;
            }
#pragma unroll
            for (int hh = 0; hh < 4; ++hh) {
              if (h0 + hh < G) {
                const float w = pr[(h0 + hh) * 64 + key];
                o0[hh] = fmaf(w, v0, o0[hh]);
                o1[hh] = fmaf(w, v1, o1[hh]);
              }
            }
          }
#pragma unroll
          for (int hh = 0; hh < 4; ++hh)
            if (h0 + hh < G) part[(kq * G + h0 + hh) * 64 + dp] = make_float2(o0[hh], o1[hh]);
        }
        named_bar_sync(1, CT);
        for (int idx = ct; idx < G * 64; idx += CT) {
          const int h = idx >> 6, d2 = idx & 63;
          float2 item = part[h * 64 + d2];
#pragma unroll
          for (int q = 1; q < 4; ++q) {
            const float2 u = part[(q * G + h) * 64 + d2];
            item.x += u.x;
            item.y += u.y;
          }
          float2* ao = reinterpret_cast<float2*>(acc_o + h * D) + d2;
          const float2 old = *ao;
          *ao = make_float2(old.x * fac[2 * h] + item.x * fac[2 * h + 1], old.y * fac[2 * h] + item.y * fac[2 * h + 1]);
        }
      }
    }
    // The stage can be refilled once every compute warp is done with it.
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[st]);
    named_bar_sync(1, CT);   // pr[] / qsum[] / acc_o[] settled for this item
    const bool seg_end = (it + 1 == it1) || ((it + 1) / p.K != bg);
    if (!seg_end) continue;
    // Segment end: one partial in the slot of its first item, empty marks in the
    // other slots it covered, then a ticket for all of its items.
    {
      float* pm = p.part_ml + ((long long)bg * p.K) * G * 2;
      float* po = p.part_o + ((long long)bg * p.K + seg_k0) * G * D;
      for (int i = ct; i < G * D; i += CT) po[i] = acc_o[i];
      for (int i = ct; i < (k - seg_k0 + 1) * G; i += CT) {
        const int kk = seg_k0 + i / G, h = i % G;
        pm[(kk * G + h) * 2] = (kk == seg_k0) ? acc_ml[2 * h] : -INFINITY;
        pm[(kk * G + h) * 2 + 1] = (kk == seg_k0) ? acc_ml[2 * h + 1] : 0.f;
      }
    }
    named_bar_sync(1, CT);
    if (ct == 0) {
      __threadfence();   // after the barrier: the whole CTA's partials precede the ticket
      const int cnt = k - seg_k0 + 1;
      const int ticket = atomicAdd(p.tickets + bg, cnt);
      *last_flag = (ticket + cnt == p.K);
    }
    named_bar_sync(1, CT);
    if (*last_flag) {
      // Merge: slot maxima and sums into shared memory, one weight per (slot, head),
      // then every output element sums the weighted slot outputs (loads unrolled).
      __threadfence();
      float* mw = qsum;                   // [K][G] weights
      float* den = qsum + p.K * G;        // [G]
      for (int i = ct; i < p.K * G; i += CT)
        mw[i] = __ldcg(p.part_ml + ((long long)bg * p.K * G + i) * 2);
      named_bar_sync(1, CT);
      for (int h = ct; h < G; h += CT) {
        float M = -INFINITY;
        for (int kk = 0; kk < p.K; ++kk) M = fmaxf(M, mw[kk * G + h]);
        float dsum = 0.f;
        for (int kk = 0; kk < p.K; ++kk) {
          const float mk = mw[kk * G + h];
          const float wgt = (mk == -INFINITY) ? 0.f : expf(mk - M);
          dsum += wgt * __ldcg(p.part_ml + (((long long)bg * p.K + kk) * G + h) * 2 + 1);
          mw[kk * G + h] = wgt;
        }
        den[h] = dsum;
      }
      named_bar_sync(1, CT);
      for (int idx = ct; idx < G * D; idx += CT) {
        const int h = idx / D, dd = idx % D;
        float num = 0.f;
#pragma unroll 4
        for (int kk = 0; kk < p.K; ++kk) {
          const float wgt = mw[kk * G + h];
          if (wgt != 0.f) num += wgt * __ldcg(p.part_o + (((long long)bg * p.K + kk) * G + h) * D + dd);
        }
        const float out = num / den[h];
        const long long oi = ((long long)b * p.Hq + g * G + h) * D + dd;
        if constexpr (sizeof(T) == 2)
          static_cast<__nv_bfloat16*>(p.o)[oi] = __float2bfloat16_rn(out);
        else
          static_cast<float*>(p.o)[oi] = out;
      }
      if (ct == 0) p.tickets[bg] = 0;   // ready for the next call
      named_bar_sync(1, CT);
    }
  }
}

size_t smem_bytes(int dtype, int G) {
  const size_t el = dtype == 1 ? 2 : 4;
  return NS * 2 * 64 * D * el + ((size_t)G * D + G * 64 + 4 * G * D + G * D + 6 * G) * 4 + 2 * NS * 8 + 16 + 128;
}

}  // namespace decode

static size_t a256(size_t x) { return (x + 255) / 256 * 256; }

size_t decode_workspace_bytes(int B, int Hq, int Hkv, int K) {
  const int G = Hq / Hkv;
  const size_t n_bg = (size_t)B * Hkv;
  size_t bytes = 256;                                      // status word
  bytes += a256(n_bg * K * sizeof(int32_t));               // attended lists
  bytes += a256(n_bg * sizeof(float));                     // log-gate LSE
  bytes += a256(n_bg * sizeof(int32_t));                   // tickets
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
  prm.lse_gate = reinterpret_cast<float*>(w + off);
  off += a256(n_bg * sizeof(float));
  prm.tickets = reinterpret_cast<int32_t*>(w + off);
  off += a256(n_bg * sizeof(int32_t));
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
  prm.n_items = (int)(n_bg * pb.K);
  prm.sm_scale = pb.sm_scale;
  // Tickets start at zero on every call.
  cudaError_t e = cudaMemsetAsync(prm.tickets, 0, n_bg * sizeof(int32_t), st);
  if (e != cudaSuccess) return e;
  decode_select_kernel<<<(unsigned)((n_bg + 7) / 8), 256, 0, st>>>(prm);
  count_launch();
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const unsigned grid = (unsigned)std::min<long long>((long long)prm.n_items, 2LL * sms);
  const size_t shm = smem_bytes(pb.dtype, G);
  if (pb.dtype == 1) {
    if ((e = cudaFuncSetAttribute(decode_attn_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)shm)) != cudaSuccess)
      return e;
    decode_attn_kernel<__nv_bfloat16><<<grid, THREADS, shm, st>>>(prm);
  } else {
    if ((e = cudaFuncSetAttribute(decode_attn_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)shm)) !=
        cudaSuccess)
      return e;
    decode_attn_kernel<float><<<grid, THREADS, shm, st>>>(prm);
  }
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
static void* g_scratch_addr[kMaxDevices] = {};
static std::mutex g_scratch_mutex;

// Device address of g_decode_scratch on the current device, looked up once per
// device. The host-side name is only a stand-in: the kernel must be given this
// address, never &g_decode_scratch.
static cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

}  // namespace decode_static

size_t decode_static_scratch_limit() { return decode_static::kScratchBytes; }

cudaError_t launch_decode_static(const DecodeProblem& pb, cudaStream_t st) {
  void* ws = nullptr;
  cudaError_t e = decode_static::scratch_address(&ws);
  if (e != cudaSuccess) return e;
  // The status word starts clear on every call (tickets are cleared by launch_decode).
  e = cudaMemsetAsync(ws, 0, sizeof(int32_t), st);
  if (e != cudaSuccess) return e;
  return launch_decode(pb, ws, st);
}

}  // namespace sas
