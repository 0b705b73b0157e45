// SAS gated block-sparse attention backward on sm_100a tensor cores.
//
// SAS paper (arXiv 2609.13141) Appendix E "Backward pass" (Algorithm 4):
// recompute P from the saved LSE, Delta = rowsum(O * dO), dS = P * (dP - Delta),
// and the block log-gate gradient as the per-block sum of dS over the tokens of
// each selected block (summed here over the G heads that share the gate).
//
// Three kernels, in the paper's two-pass shape:
//   delta_kernel        Delta[row] = sum_d O * dO                (HBM-bound)
//   sas_bwd_dq_kernel   q-tile outer, selected blocks inner: S = Q K^T and
//                       dP = dO V^T into TMEM, dS written back to TMEM as bf16,
//                       dQ += dS K accumulated in TMEM; dLogG from per-row sums
//                       of dS, reduced over the group's heads in shared memory.
//   sas_bwd_dkv_kernel  KV-block outer, q-tiles that use the block inner:
//                       S and dP again, P and dS written to shared memory,
//                       dV^T += dO^T P and dK^T += Q^T dS accumulated in TMEM.
#include "sas_common.cuh"
#include "sas_kernels.h"
#include "sas_tmap.h"

namespace sas {
namespace bwd {

constexpr int D = 128;
constexpr uint32_t TILE_BYTES = 128 * D * 2;   // a 128-row x 128-col bf16 tile: 2 halves of 16 KiB
constexpr uint32_t HALF128 = 128 * 128;        // one half of a 128-row tile
constexpr uint32_t KV_HALF = 64 * 128;         // one half of a 64-row tile
constexpr int MAX_NB = 4096;

struct Params {
  const float* logG;
  const float* tau;
  const int32_t* tau_idx;
  const float* LSE;
  const float* delta;
  const uint32_t* masks;
  __nv_bfloat16* dQ;
  __nv_bfloat16* dK;
  __nv_bfloat16* dV;
  float* dLogG;
  int32_t* status;
  int B, Hq, Hkv, T, NB, NBW, G, P, n_ptiles;
  float scale_log2, sm_scale;
};

// Per-row bias of one block: returns false when the whole block is masked for the row.
__device__ __forceinline__ bool row_block_bias(bool valid, int t, int c_t, int m, float gv, float tau_t, int tidx_t,
                                               int& lim, float& bias2) {
  lim = 63;
  bias2 = 0.f;
  if (!valid) return false;
  if (m == c_t) {
    lim = t - m * kBlock;
    return true;
  }
  if (m < c_t && (gv > tau_t || (gv == tau_t && m <= tidx_t))) {
    bias2 = gv * kLog2e;
    return true;
  }
  return false;
}

// ============================================================================ Delta
__global__ void __launch_bounds__(256) delta_kernel(const __nv_bfloat16* __restrict__ O,
                                                    const __nv_bfloat16* __restrict__ dO, float* __restrict__ delta,
                                                    long long rows) {
  const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const uint2 a = *reinterpret_cast<const uint2*>(O + row * D + lane * 4);
  const uint2 c = *reinterpret_cast<const uint2*>(dO + row * D + lane * 4);
  const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a);
  const __nv_bfloat162* c2 = reinterpret_cast<const __nv_bfloat162*>(&c);
  float acc = 0.f;
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const float2 x = __bfloat1622float2(a2[i]);
    const float2 y = __bfloat1622float2(c2[i]);
    acc = fmaf(x.x, y.x, acc);
    acc = fmaf(x.y, y.y, acc);
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) delta[row] = acc;
}

// ============================================================================ dQ + dLogG
namespace dq {
constexpr int NST = 3;
constexpr int THREADS = 192;
constexpr uint32_t STAGE_BYTES = 4 * KV_HALF;   // K + V of one block
constexpr uint32_t OFF_DO = TILE_BYTES;
constexpr uint32_t OFF_KV = 2 * TILE_BYTES;
constexpr uint32_t OFF_BAR = OFF_KV + NST * STAGE_BYTES;
constexpr uint32_t OFF_MISC = OFF_BAR + 256;
constexpr uint32_t OFF_RED = OFF_MISC + 64;     // 2 x 128 floats
constexpr uint32_t OFF_LIST = OFF_RED + 2 * 128 * 4;
constexpr uint32_t OFF_WORDS = OFF_LIST + MAX_NB * 2;
constexpr uint32_t SMEM_BYTES = OFF_WORDS + (MAX_NB / 32) * 4 + 1024;
constexpr uint32_t COL_DQ = 0, COL_S0 = 128, COL_DP0 = 256, COL_DS0 = 384, TMEM_COLS = 512;

struct Bars {
  uint64_t q_full, k_full[NST], v_full[NST], kv_empty[NST], s_full[2], ds_full[2], dq_done[2], fin;
};

__global__ void __launch_bounds__(THREADS, 1)
    sas_bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmdO,
                      const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                      const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars* bars = reinterpret_cast<Bars*>(smem + OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_MISC);
  int* n_list_s = reinterpret_cast<int*>(smem + OFF_MISC + 8);
  float* red = reinterpret_cast<float*>(smem + OFF_RED);
  uint16_t* list = reinterpret_cast<uint16_t*>(smem + OFF_LIST);
  uint32_t* words = reinterpret_cast<uint32_t*>(smem + OFF_WORDS);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nbg = p.B * p.Hkv;
  const int bg = blockIdx.x % nbg;
  const int pt = p.n_ptiles - 1 - blockIdx.x / nbg;
  const int b = bg / p.Hkv, g = bg % p.Hkv;
  const int t0 = pt * p.P;
  const int t_end = min(t0 + p.P, p.T);
  const int cur_lo = t0 / kBlock, cur_hi = (t_end - 1) / kBlock;
  const int rows_used = p.G * p.P;
  int32_t* status = p.status;

  if (warp == 5) tmem_alloc(tmem_slot, TMEM_COLS);
  if (tid == 0) {
    mbar_init(&bars->q_full, 1);
    for (int i = 0; i < NST; ++i) {
      mbar_init(&bars->k_full[i], 1);
      mbar_init(&bars->v_full[i], 1);
      mbar_init(&bars->kv_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->s_full[i], 1);
      mbar_init(&bars->ds_full[i], 4);
      mbar_init(&bars->dq_done[i], 1);
    }
    mbar_init(&bars->fin, 1);
    fence_barrier_init();
  }
  if (rows_used < 128) {
    const int per = (128 - rows_used) * 8;
    for (int i = tid; i < per * 4; i += THREADS) {
      const int tile = i / (2 * per);   // 0 = Q, 1 = dO
      const int half = (i / per) & 1;
      const int rem = i % per;
      *reinterpret_cast<uint4*>(smem + tile * TILE_BYTES + half * HALF128 + (rows_used + rem / 8) * 128 +
                                (rem % 8) * 16) = make_uint4(0, 0, 0, 0);
    }
    fence_proxy_async_smem();
  }
  const uint32_t* tile_mask = p.masks + ((long long)bg * p.n_ptiles + pt) * p.NBW;
  for (int w = tid; w < p.NBW; w += THREADS) words[w] = tile_mask[w];
  __syncthreads();
  if (warp == 0) {
    int base = 0;
    if (lane == 0)
      for (int m = cur_hi; m >= cur_lo; --m) list[base++] = (uint16_t)m;
    base = __shfl_sync(0xffffffffu, base, 0);
    for (int w0 = p.NBW - 1; w0 >= 0; w0 -= 32) {
      const int w = w0 - lane;
      uint32_t bits = 0u;
      if (w >= 0) {
        bits = words[w];
        const int lo = w * 32;
        if (lo + 32 > cur_lo)
          bits &= (cur_lo - lo <= 0) ? 0u : ((cur_lo - lo >= 32) ? 0xffffffffu : ((1u << (cur_lo - lo)) - 1u));
      }
      const int cnt = __popc(bits);
      int incl = cnt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      int pos = base + incl - cnt;
      while (bits) {
        const int hb = 31 - __clz(bits);
        list[pos++] = (uint16_t)(w * 32 + hb);
        bits &= ~(1u << hb);
      }
      base += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) *n_list_s = base;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int n = *n_list_s;
  const uint32_t s_base = smem_u32(smem);

  if (warp == 4) {
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmdO);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      mbar_expect_tx(&bars->q_full, (uint32_t)(2 * p.G * p.P * 128 * 2));
      for (int hh = 0; hh < p.G; ++hh)
        for (int half = 0; half < 2; ++half) {
          const int zq = b * p.Hq + g * p.G + hh;
          tma_load_3d(smem + half * HALF128 + hh * p.P * 128, &tmQ, &bars->q_full, half * 64, t0, zq);
          tma_load_3d(smem + OFF_DO + half * HALF128 + hh * p.P * 128, &tmdO, &bars->q_full, half * 64, t0, zq);
        }
      int issued = 0;
      for (int j = 0; j < n; ++j) {
        const int st = j % NST;
        if (j >= NST && !mbar_wait(&bars->kv_empty[st], ((j / NST) - 1) & 1, status)) break;
        const int m = list[j];
        uint8_t* kv = smem + OFF_KV + st * STAGE_BYTES;
        mbar_expect_tx(&bars->k_full[st], 2 * KV_HALF);
        tma_load_3d(kv, &tmK, &bars->k_full[st], 0, m * kBlock, b * p.Hkv + g);
        tma_load_3d(kv + KV_HALF, &tmK, &bars->k_full[st], 64, m * kBlock, b * p.Hkv + g);
        mbar_expect_tx(&bars->v_full[st], 2 * KV_HALF);
        tma_load_3d(kv + 2 * KV_HALF, &tmV, &bars->v_full[st], 0, m * kBlock, b * p.Hkv + g);
        tma_load_3d(kv + 3 * KV_HALF, &tmV, &bars->v_full[st], 64, m * kBlock, b * p.Hkv + g);
        issued = j + 1;
      }
      for (int j = max(0, issued - NST); j < issued; ++j) {
        mbar_wait_drain(&bars->k_full[j % NST], (j / NST) & 1);
        mbar_wait_drain(&bars->v_full[j % NST], (j / NST) & 1);
      }
      mbar_wait_drain(&bars->q_full, 0);
    }
  } else if (warp == 5) {
    if (lane == 0) {
      const uint32_t idesc_s = make_idesc_bf16(128, 64, 0, 0);
      const uint32_t idesc_dq = make_idesc_bf16(128, D, 0, 1);
      bool ok = mbar_wait(&bars->q_full, 0, status);
      for (int j = 0; ok && j <= n; ++j) {
        if (j < n) {
          const int st = j % NST, sb = j & 1;
          ok = mbar_wait(&bars->k_full[st], (j / NST) & 1, status);
          if (ok) ok = mbar_wait(&bars->v_full[st], (j / NST) & 1, status);
          if (ok && j >= 2) ok = mbar_wait(&bars->ds_full[sb], ((j - 2) >> 1) & 1, status);
          if (!ok) break;
          tc_fence_after();
          const uint32_t kb = s_base + OFF_KV + st * STAGE_BYTES;
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks) {
            const uint32_t half = ks >> 2, koff = (ks & 3) * 32;
            const uint64_t aq = make_sdesc(s_base + half * HALF128 + koff, 16, 1024);
            const uint64_t bk = make_sdesc(kb + half * KV_HALF + koff, 16, 1024);
            umma_ss(tmem + COL_S0 + 64 * sb, aq, bk, idesc_s, ks > 0 ? 1u : 0u);
          }
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks) {
            const uint32_t half = ks >> 2, koff = (ks & 3) * 32;
            const uint64_t ado = make_sdesc(s_base + OFF_DO + half * HALF128 + koff, 16, 1024);
            const uint64_t bv = make_sdesc(kb + 2 * KV_HALF + half * KV_HALF + koff, 16, 1024);
            umma_ss(tmem + COL_DP0 + 64 * sb, ado, bv, idesc_s, ks > 0 ? 1u : 0u);
          }
          umma_commit(&bars->s_full[sb]);
        }
        if (j >= 1) {
          const int jj = j - 1, st = jj % NST, pb = jj & 1;
          ok = mbar_wait(&bars->ds_full[pb], (jj >> 1) & 1, status);
          if (!ok) break;
          tc_fence_after();
          const uint32_t kb = s_base + OFF_KV + st * STAGE_BYTES;
#pragma unroll
          for (int ks = 0; ks < 4; ++ks) {
            const uint64_t bk = make_sdesc(kb + ks * 2048, KV_HALF, 1024);
            umma_ts(tmem + COL_DQ, tmem + COL_DS0 + 32 * pb + ks * 8, bk, idesc_dq, (jj > 0 || ks > 0) ? 1u : 0u);
          }
          umma_commit(&bars->dq_done[pb]);
          umma_commit(&bars->kv_empty[st]);
        }
      }
      umma_commit(&bars->fin);
      mbar_wait_drain(&bars->fin, 0);
    }
  } else {
    const int r = tid;
    const int hh = r / p.P, pp = r % p.P;
    const int t = t0 + pp;
    const bool valid = (r < rows_used) && (t < p.T);
    const int c_t = valid ? t / kBlock : -1;
    const long long grow = (long long)bg * p.T + (valid ? t : 0);
    const int h = g * p.G + (valid ? hh : 0);
    const long long qrow = ((long long)b * p.Hq + h) * p.T + (valid ? t : 0);
    const float tau_t = valid ? p.tau[grow] : INFINITY;
    const int tidx_t = valid ? p.tau_idx[grow] : -1;
    const float lse2 = valid ? p.LSE[qrow] * kLog2e : 0.f;
    const float dlt = valid ? p.delta[qrow] : 0.f;
    const float* gate_row = p.logG + grow * (long long)p.NB;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    bool ok = true;
    float gate_next = 0.f;
    if (n > 0) gate_next = (valid && list[0] < c_t) ? __ldg(gate_row + list[0]) : 0.f;
    for (int j = 0; j < n; ++j) {
      const int m = list[j];
      const int sb = j & 1;
      const float gv = gate_next;
      if (j + 1 < n) gate_next = (valid && list[j + 1] < c_t) ? __ldg(gate_row + list[j + 1]) : 0.f;
      int lim;
      float bias2;
      const bool active = row_block_bias(valid, t, c_t, m, gv, tau_t, tidx_t, lim, bias2);
      const bool hist_sel = active && (m != c_t);
      bool step_ok = warp_wait(&bars->s_full[sb], (j >> 1) & 1, status);
      uint32_t sr[2][32], dr[2][32];
      if (step_ok) {
        tc_fence_after();
        tmem_ld32(tmem + lane_base + COL_S0 + 64 * sb, sr[0]);
        tmem_ld32(tmem + lane_base + COL_S0 + 64 * sb + 32, sr[1]);
        tmem_ld32(tmem + lane_base + COL_DP0 + 64 * sb, dr[0]);
        tmem_ld32(tmem + lane_base + COL_DP0 + 64 * sb + 32, dr[1]);
        tmem_wait_ld();
      }
      if (step_ok && j >= 2) step_ok = warp_wait(&bars->dq_done[sb], ((j - 2) >> 1) & 1, status);
      float rs = 0.f;
      if (step_ok) {
        uint32_t pk[32];
#pragma unroll
        for (int k = 0; k < 32; ++k) {
          float ds2[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int kk = 2 * k + e;
            const float sv = __uint_as_float(sr[kk >> 5][kk & 31]);
            const float dp = __uint_as_float(dr[kk >> 5][kk & 31]);
            const float pr = (active && kk <= lim) ? ex2(fmaf(sv, p.scale_log2, bias2) - lse2) : 0.f;
            ds2[e] = pr * (dp - dlt);
            rs += ds2[e];
          }
          pk[k] = pack_bf16(ds2[0], ds2[1]);
        }
        tmem_st32(tmem + lane_base + COL_DS0 + 32 * sb, pk);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->ds_full[sb]);
      }
      // dLogG[t, m]: sum over the G heads of this position's row sums (rows
      // hh * P + pp hold head hh of position pp). The barrier also agrees on
      // success across the four softmax warps so that none is left waiting.
      red[sb * 128 + r] = hist_sel ? rs : 0.f;
      ok = named_bar_and(1, 128, step_ok);
      if (!ok) break;
      if (r < p.P && hist_sel) {   // r < P: head 0 of position pp = r, selection shared by the heads
        float acc = 0.f;
        for (int q = 0; q < p.G; ++q) acc += red[sb * 128 + q * p.P + r];
        p.dLogG[grow * (long long)p.NB + m] = acc;
      }
    }
    if (ok && n > 0) ok = warp_wait(&bars->dq_done[(n - 1) & 1], ((n - 1) >> 1) & 1, status);
    if (ok) {
      tc_fence_after();
      __nv_bfloat16* drow = p.dQ + qrow * D;
#pragma unroll 1
      for (int ch = 0; ch < D / 32; ++ch) {
        uint32_t o[32];
        tmem_ld32(tmem + lane_base + COL_DQ + 32 * ch, o);
        tmem_wait_ld();
        if (valid) {
          uint32_t w[16];
#pragma unroll
          for (int k = 0; k < 16; ++k)
            w[k] = pack_bf16(__uint_as_float(o[2 * k]) * p.sm_scale, __uint_as_float(o[2 * k + 1]) * p.sm_scale);
          uint4* dst = reinterpret_cast<uint4*>(drow + 32 * ch);
#pragma unroll
          for (int k = 0; k < 4; ++k) dst[k] = make_uint4(w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}
}  // namespace dq

// ============================================================================ dK / dV
namespace dkv {
constexpr int NST = 2;                          // Q/dO ring stages
constexpr int THREADS = 192;
constexpr uint32_t STAGE_BYTES = 2 * TILE_BYTES;   // Q tile + dO tile
constexpr uint32_t OFF_K = 0;                   // K_j: 2 halves of [64 rows][128 B]
constexpr uint32_t OFF_V = 2 * KV_HALF;
constexpr uint32_t OFF_QD = 4 * KV_HALF;
constexpr uint32_t OFF_P = OFF_QD + NST * STAGE_BYTES;   // P tile [128 rows][64 keys] bf16, 16 KiB
constexpr uint32_t OFF_DS = OFF_P + 128 * 128;           // dS tile, 16 KiB
constexpr uint32_t OFF_BAR = OFF_DS + 128 * 128;
constexpr uint32_t OFF_MISC = OFF_BAR + 256;
constexpr int MAX_QT = 8192;
constexpr uint32_t OFF_LIST = OFF_MISC + 64;
constexpr uint32_t SMEM_BYTES = OFF_LIST + MAX_QT * 2 + 1024;
constexpr uint32_t COL_S = 0, COL_DP = 64, COL_DV = 128, COL_DK = 192, TMEM_COLS = 256;

struct Bars {
  uint64_t kv_full, qd_full[NST], qd_empty[NST], s_full, p_full, pd_free, fin;
};

__global__ void __launch_bounds__(THREADS, 1)
    sas_bwd_dkv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmdO,
                       const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                       const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars* bars = reinterpret_cast<Bars*>(smem + OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_MISC);
  int* n_list_s = reinterpret_cast<int*>(smem + OFF_MISC + 8);
  uint16_t* list = reinterpret_cast<uint16_t*>(smem + OFF_LIST);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nbg = p.B * p.Hkv;
  const int bg = blockIdx.x % nbg;
  const int jb = blockIdx.x / nbg;   // KV block; small j (most rows attend it) first
  const int b = bg / p.Hkv, g = bg % p.Hkv;
  const int rows_used = p.G * p.P;
  int32_t* status = p.status;

  if (warp == 5) tmem_alloc(tmem_slot, TMEM_COLS);
  if (tid == 0) {
    mbar_init(&bars->kv_full, 1);
    for (int i = 0; i < NST; ++i) {
      mbar_init(&bars->qd_full[i], 1);
      mbar_init(&bars->qd_empty[i], 1);
    }
    mbar_init(&bars->s_full, 1);
    mbar_init(&bars->p_full, 4);
    mbar_init(&bars->pd_free, 1);
    mbar_init(&bars->fin, 1);
    fence_barrier_init();
  }
  if (rows_used < 128) {
    const int per = (128 - rows_used) * 8;
    for (int i = tid; i < per * 2 * 2 * NST; i += THREADS) {
      const int tile = i / (2 * per);   // stage * 2 + (0 = Q, 1 = dO)
      const int half = (i / per) & 1;
      const int rem = i % per;
      *reinterpret_cast<uint4*>(smem + OFF_QD + tile * TILE_BYTES + half * HALF128 + (rows_used + rem / 8) * 128 +
                                (rem % 8) * 16) = make_uint4(0, 0, 0, 0);
    }
    fence_proxy_async_smem();
  }
  // q-tiles that use block jb: those overlapping the block's own positions, and
  // later ones whose union mask has bit jb.
  if (warp == 0) {
    const int pt_first = (jb * kBlock) / p.P;
    const int own_last = min((jb * kBlock + kBlock - 1) / p.P, p.n_ptiles - 1);
    int base = 0;
    for (int c0 = pt_first; c0 < p.n_ptiles; c0 += 32) {
      const int ptl = c0 + lane;
      bool use = false;
      if (ptl < p.n_ptiles) {
        use = ptl <= own_last;
        if (!use) use = (p.masks[((long long)bg * p.n_ptiles + ptl) * p.NBW + (jb >> 5)] >> (jb & 31)) & 1u;
      }
      const uint32_t bal = __ballot_sync(0xffffffffu, use);
      if (use) list[base + __popc(bal & ((1u << lane) - 1u))] = (uint16_t)ptl;
      base += __popc(bal);
    }
    if (lane == 0) *n_list_s = base;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int n = *n_list_s;
  const uint32_t s_base = smem_u32(smem);

  if (warp == 4) {
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmdO);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      mbar_expect_tx(&bars->kv_full, 4 * KV_HALF);
      tma_load_3d(smem + OFF_K, &tmK, &bars->kv_full, 0, jb * kBlock, b * p.Hkv + g);
      tma_load_3d(smem + OFF_K + KV_HALF, &tmK, &bars->kv_full, 64, jb * kBlock, b * p.Hkv + g);
      tma_load_3d(smem + OFF_V, &tmV, &bars->kv_full, 0, jb * kBlock, b * p.Hkv + g);
      tma_load_3d(smem + OFF_V + KV_HALF, &tmV, &bars->kv_full, 64, jb * kBlock, b * p.Hkv + g);
      int issued = 0;
      for (int i = 0; i < n; ++i) {
        const int st = i % NST;
        if (i >= NST && !mbar_wait(&bars->qd_empty[st], ((i / NST) - 1) & 1, status)) break;
        const int t0 = list[i] * p.P;
        uint8_t* qd = smem + OFF_QD + st * STAGE_BYTES;
        mbar_expect_tx(&bars->qd_full[st], (uint32_t)(2 * p.G * p.P * 128 * 2));
        for (int hh = 0; hh < p.G; ++hh)
          for (int half = 0; half < 2; ++half) {
            const int zq = b * p.Hq + g * p.G + hh;
            tma_load_3d(qd + half * HALF128 + hh * p.P * 128, &tmQ, &bars->qd_full[st], half * 64, t0, zq);
            tma_load_3d(qd + TILE_BYTES + half * HALF128 + hh * p.P * 128, &tmdO, &bars->qd_full[st], half * 64,
                        t0, zq);
          }
        issued = i + 1;
      }
      for (int i = max(0, issued - NST); i < issued; ++i) mbar_wait_drain(&bars->qd_full[i % NST], (i / NST) & 1);
      mbar_wait_drain(&bars->kv_full, 0);
    }
  } else if (warp == 5) {
    if (lane == 0) {
      const uint32_t idesc_s = make_idesc_bf16(128, 64, 0, 0);
      const uint32_t idesc_t = make_idesc_bf16(128, 64, 1, 1);   // (d x rows) * (rows x keys), both MN-major
      bool ok = mbar_wait(&bars->kv_full, 0, status);
      for (int i = 0; ok && i < n; ++i) {
        const int st = i % NST;
        ok = mbar_wait(&bars->qd_full[st], (i / NST) & 1, status);
        // S/dP in TMEM are free once the softmax warps consumed tile i-1 (p_full of i-1).
        if (ok && i >= 1) ok = mbar_wait(&bars->p_full, (i - 1) & 1, status);
        if (!ok) break;
        tc_fence_after();
        const uint32_t qb = s_base + OFF_QD + st * STAGE_BYTES;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t half = ks >> 2, koff = (ks & 3) * 32;
          umma_ss(tmem + COL_S, make_sdesc(qb + half * HALF128 + koff, 16, 1024),
                  make_sdesc(s_base + OFF_K + half * KV_HALF + koff, 16, 1024), idesc_s, ks > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t half = ks >> 2, koff = (ks & 3) * 32;
          umma_ss(tmem + COL_DP, make_sdesc(qb + TILE_BYTES + half * HALF128 + koff, 16, 1024),
                  make_sdesc(s_base + OFF_V + half * KV_HALF + koff, 16, 1024), idesc_s, ks > 0 ? 1u : 0u);
        }
        umma_commit(&bars->s_full);
        ok = mbar_wait(&bars->p_full, i & 1, status);
        if (!ok) break;
        tc_fence_after();
        // dV^T (d x keys) += dO^T P ; dK^T += Q^T dS ; K dimension = the tile's 128 rows.
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint64_t a_do = make_sdesc(qb + TILE_BYTES + ks * 2048, HALF128, 1024);
          const uint64_t b_p = make_sdesc(s_base + OFF_P + ks * 2048, HALF128, 1024);
          umma_ss(tmem + COL_DV, a_do, b_p, idesc_t, (i > 0 || ks > 0) ? 1u : 0u);
        }
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint64_t a_q = make_sdesc(qb + ks * 2048, HALF128, 1024);
          const uint64_t b_ds = make_sdesc(s_base + OFF_DS + ks * 2048, HALF128, 1024);
          umma_ss(tmem + COL_DK, a_q, b_ds, idesc_t, (i > 0 || ks > 0) ? 1u : 0u);
        }
        umma_commit(&bars->pd_free);
        umma_commit(&bars->qd_empty[st]);
      }
      umma_commit(&bars->fin);
      mbar_wait_drain(&bars->fin, 0);
    }
  } else {
    const int r = tid;
    const int hh = r / p.P, pp = r % p.P;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    bool ok = true;
    // Row metadata of the next tile, loaded one tile ahead.
    auto load_meta = [&](int i, bool& valid, int& t, float& tau_t, int& tidx_t, float& lse2, float& dlt,
                         float& gv) {
      t = list[i] * p.P + pp;
      valid = (r < rows_used) && (t < p.T);
      const long long grow = (long long)bg * p.T + (valid ? t : 0);
      const long long qrow = ((long long)b * p.Hq + g * p.G + (valid ? hh : 0)) * p.T + (valid ? t : 0);
      tau_t = valid ? p.tau[grow] : INFINITY;
      tidx_t = valid ? p.tau_idx[grow] : -1;
      lse2 = valid ? p.LSE[qrow] * kLog2e : 0.f;
      dlt = valid ? p.delta[qrow] : 0.f;
      gv = (valid && jb < t / kBlock) ? p.logG[grow * (long long)p.NB + jb] : 0.f;
    };
    bool nvalid = false;
    int nt = 0, ntidx = -1;
    float ntau = 0.f, nlse2 = 0.f, ndlt = 0.f, ngv = 0.f;
    if (n > 0) load_meta(0, nvalid, nt, ntau, ntidx, nlse2, ndlt, ngv);
    for (int i = 0; i < n; ++i) {
      const bool valid = nvalid;
      const int t = nt, tidx_t = ntidx;
      const float tau_t = ntau, lse2 = nlse2, dlt = ndlt, gv = ngv;
      if (i + 1 < n) load_meta(i + 1, nvalid, nt, ntau, ntidx, nlse2, ndlt, ngv);
      int lim;
      float bias2;
      const bool active = row_block_bias(valid, t, valid ? t / kBlock : -1, jb, gv, tau_t, tidx_t, lim, bias2);
      ok = warp_wait(&bars->s_full, i & 1, status);
      if (!ok) break;
      tc_fence_after();
      uint32_t sr[2][32], dr[2][32];
      tmem_ld32(tmem + lane_base + COL_S, sr[0]);
      tmem_ld32(tmem + lane_base + COL_S + 32, sr[1]);
      tmem_ld32(tmem + lane_base + COL_DP, dr[0]);
      tmem_ld32(tmem + lane_base + COL_DP + 32, dr[1]);
      tmem_wait_ld();
      // The P / dS tiles in shared memory are free once tile i-1's dV/dK MMAs completed.
      if (i >= 1) {
        ok = warp_wait(&bars->pd_free, (i - 1) & 1, status);
        if (!ok) break;
      }
      uint8_t* prow = smem + OFF_P;
      uint8_t* srow = smem + OFF_DS;
#pragma unroll
      for (int ch = 0; ch < 8; ++ch) {
        uint32_t pw[4], sw[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          float pv[2], dv[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int kk = ch * 8 + 2 * k + e;
            const float sv = __uint_as_float(sr[kk >> 5][kk & 31]);
            const float dp = __uint_as_float(dr[kk >> 5][kk & 31]);
            pv[e] = (active && kk <= lim) ? ex2(fmaf(sv, p.scale_log2, bias2) - lse2) : 0.f;
            dv[e] = pv[e] * (dp - dlt);
          }
          pw[k] = pack_bf16(pv[0], pv[1]);
          sw[k] = pack_bf16(dv[0], dv[1]);
        }
        const uint32_t off = sw128_offset((uint32_t)r, (uint32_t)ch);
        *reinterpret_cast<uint4*>(prow + off) = make_uint4(pw[0], pw[1], pw[2], pw[3]);
        *reinterpret_cast<uint4*>(srow + off) = make_uint4(sw[0], sw[1], sw[2], sw[3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->p_full);
    }
    if (ok && n > 0) ok = warp_wait(&bars->pd_free, (n - 1) & 1, status);
    if (ok) {
      tc_fence_after();
      // TMEM lane = feature index dd, column = key within the block.
      const int dd = r;
      const long long key0 = ((long long)b * p.Hkv + g) * p.T + (long long)jb * kBlock;
#pragma unroll 1
      for (int which = 0; which < 2; ++which) {
        const uint32_t col = which == 0 ? COL_DV : COL_DK;
        __nv_bfloat16* dst = which == 0 ? p.dV : p.dK;
        const float scl = which == 0 ? 1.f : p.sm_scale;
#pragma unroll 1
        for (int ch = 0; ch < 2; ++ch) {
          uint32_t o[32];
          tmem_ld32(tmem + lane_base + col + 32 * ch, o);
          tmem_wait_ld();
          if (n > 0) {
#pragma unroll
            for (int k = 0; k < 32; ++k)
              dst[(key0 + 32 * ch + k) * D + dd] = __float2bfloat16_rn(__uint_as_float(o[k]) * scl);
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}
}  // namespace dkv

}  // namespace bwd

cudaError_t launch_bwd_tc(const TcProblem& pb, void* dQ, void* dK, void* dV, float* dLogG, int32_t* status,
                          uint32_t* masks, float* delta, cudaStream_t st) {
  const QTileShape qs = qtile_shape(pb.G, pb.T, pb.NB);
  const long long qrows = (long long)pb.B * pb.Hq * pb.T;
  cudaError_t e = cudaMemsetAsync(dLogG, 0, (size_t)pb.B * pb.Hkv * pb.T * pb.NB * sizeof(float), st);
  if (e != cudaSuccess) return e;
  bwd::delta_kernel<<<(unsigned)((qrows + 7) / 8), 256, 0, st>>>(
      reinterpret_cast<const __nv_bfloat16*>(pb.O), reinterpret_cast<const __nv_bfloat16*>(pb.dO), delta, qrows);
  count_launch();
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  e = launch_tile_union(pb.logG, pb.tau, pb.tau_idx, masks, (long long)pb.B * pb.Hkv, pb.T, pb.NB, qs.P,
                        qs.n_ptiles, qs.NBW, st);
  if (e != cudaSuccess) return e;
  CUtensorMap tq, tdo, tk, tv;
  if (!make_tmap_bf16_3d(&tq, pb.Q, pb.d, pb.T, (uint64_t)pb.B * pb.Hq, qs.P) ||
      !make_tmap_bf16_3d(&tdo, pb.dO, pb.d, pb.T, (uint64_t)pb.B * pb.Hq, qs.P) ||
      !make_tmap_bf16_3d(&tk, pb.K, pb.d, pb.T, (uint64_t)pb.B * pb.Hkv, 64) ||
      !make_tmap_bf16_3d(&tv, pb.V, pb.d, pb.T, (uint64_t)pb.B * pb.Hkv, 64))
    return cudaErrorInvalidValue;
  bwd::Params prm;
  prm.logG = pb.logG;
  prm.tau = pb.tau;
  prm.tau_idx = pb.tau_idx;
  prm.LSE = pb.LSE;
  prm.delta = delta;
  prm.masks = masks;
  prm.dQ = reinterpret_cast<__nv_bfloat16*>(dQ);
  prm.dK = reinterpret_cast<__nv_bfloat16*>(dK);
  prm.dV = reinterpret_cast<__nv_bfloat16*>(dV);
  prm.dLogG = dLogG;
  prm.status = status;
  prm.B = pb.B;
  prm.Hq = pb.Hq;
  prm.Hkv = pb.Hkv;
  prm.T = pb.T;
  prm.NB = pb.NB;
  prm.NBW = qs.NBW;
  prm.G = pb.G;
  prm.P = qs.P;
  prm.n_ptiles = qs.n_ptiles;
  prm.scale_log2 = pb.sm_scale * kLog2e;
  prm.sm_scale = pb.sm_scale;
  e = cudaFuncSetAttribute(bwd::dq::sas_bwd_dq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           bwd::dq::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(bwd::dkv::sas_bwd_dkv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           bwd::dkv::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  const unsigned grid_dq = (unsigned)((long long)pb.B * pb.Hkv * qs.n_ptiles);
  bwd::dq::sas_bwd_dq_kernel<<<grid_dq, bwd::dq::THREADS, bwd::dq::SMEM_BYTES, st>>>(tq, tdo, tk, tv, prm);
  count_launch();
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const unsigned grid_dkv = (unsigned)((long long)pb.B * pb.Hkv * pb.NB);
  bwd::dkv::sas_bwd_dkv_kernel<<<grid_dkv, bwd::dkv::THREADS, bwd::dkv::SMEM_BYTES, st>>>(tq, tdo, tk, tv, prm);
  count_launch();
  return cudaGetLastError();
}

}  // namespace sas
