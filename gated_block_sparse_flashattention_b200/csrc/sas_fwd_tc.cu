// SAS gated block-sparse attention forward on sm_100a tensor cores.
//
// SAS paper (arXiv 2609.13141) §4.3 eq. 9 and Appendix E "Forward pass": a
// FlashAttention-style scan over the key/value blocks a query tile needs; the
// current block is causal and unbiased, a selected historical block gets the
// row's log gate added to its logits, a non-selected one is masked, and a block
// no row of the tile selects is never loaded.
//
// Tile: 128 TMEM lanes = G heads x P consecutive positions of one (b, g) (the
// heads share the selection, so packing them adds no extra blocks). Warp roles:
//   warps 0-3  softmax: one thread per row; gate bias, threshold mask, online
//              softmax (exp2 domain), P written back to TMEM as bf16, epilogue;
//   warp 4     TMA producer: Q tile once, then K/V of each block of the tile's
//              block list into a 2-stage ring;
//   warp 5     MMA issuer (one thread): S = Q K^T (M=128, N=64, K=128) into a
//              double-buffered TMEM S, O += P V (A = P from TMEM, N=128) into
//              the TMEM O accumulator. Also owns the TMEM allocation.
// Two CTAs share an SM (256 TMEM columns and about 107 KB of shared memory
// each), so one tile's softmax runs while the other's waits on its MMAs. P is
// written over the first half of its S buffer; S of block j+2 reuses that buffer
// only after the P V of block j has completed.
#include "sas_common.cuh"
#include "sas_kernels.h"
#include "sas_tmap.h"

namespace sas {
namespace fwd {

constexpr int D = 128;
constexpr int NST = 2;                      // K/V ring stages
constexpr int THREADS = 192;
constexpr uint32_t Q_BYTES = 128 * D * 2;   // 32 KiB: 2 halves of [128 rows][128 B]
constexpr uint32_t KV_HALF = 64 * 128;      // one 64-row x 128-byte half tile (8 KiB)
constexpr uint32_t STAGE_BYTES = 4 * KV_HALF;   // K (2 halves) + V (2 halves)
constexpr uint32_t OFF_KV = Q_BYTES;
constexpr uint32_t OFF_BAR = OFF_KV + NST * STAGE_BYTES;
constexpr uint32_t OFF_MISC = OFF_BAR + 256;
constexpr uint32_t OFF_LIST = OFF_MISC + 64;
constexpr int MAX_NB = 4096;
constexpr uint32_t OFF_WORDS = OFF_LIST + MAX_NB * 2;
constexpr uint32_t SMEM_BYTES = OFF_WORDS + (MAX_NB / 32) * 4 + 1024;   // +1024 alignment slack

// TMEM columns.
constexpr uint32_t COL_O = 0;
constexpr uint32_t COL_S0 = 128;    // S buffers: 128 + 64*sb
// P (bf16 pairs) of block j goes over the first 32 columns of S buffer j & 1.
constexpr uint32_t TMEM_COLS = 256;
constexpr float RESCALE_THRESHOLD = 8.0f;   // log2 units: rescale O only when the max grows by > 2^8

struct Params {
  const float* logG;       // log gates, or raw scores when gate_lse is set
  const float* gate_lse;   // null, or the LSE of each row's historical scores
  const float* tau;
  const int32_t* tau_idx;
  const uint32_t* masks;
  __nv_bfloat16* O;
  float* LSE;
  int32_t* status;
  int B, Hq, Hkv, T, NB, NBW, G, P, n_ptiles;
  float scale_log2;
  uint64_t wait_ns;
};

struct Bars {
  uint64_t q_full, k_full[NST], v_full[NST], kv_empty[NST], s_full[2], p_full[2], pv_done[2], fin;
};

__global__ void __launch_bounds__(THREADS, 2)
    sas_fwd_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars* bars = reinterpret_cast<Bars*>(smem + OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_MISC);
  int* n_list_s = reinterpret_cast<int*>(smem + OFF_MISC + 8);
  uint16_t* list = reinterpret_cast<uint16_t*>(smem + OFF_LIST);
  uint32_t* words = reinterpret_cast<uint32_t*>(smem + OFF_WORDS);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int nbg = p.B * p.Hkv;
  const int bg = blockIdx.x % nbg;
  const int pt = p.n_ptiles - 1 - blockIdx.x / nbg;   // longest rows first
  const int b = bg / p.Hkv;
  const int g = bg % p.Hkv;
  const int t0 = pt * p.P;
  const int t_end = min(t0 + p.P, p.T);
  const int cur_lo = t0 / kBlock;
  const int cur_hi = (t_end - 1) / kBlock;
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
      mbar_init(&bars->p_full[i], 4);
      mbar_init(&bars->pv_done[i], 1);
    }
    mbar_init(&bars->fin, 1);
    fence_barrier_init();
  }
  // Rows beyond G*P of the Q tile are never loaded: zero them once.
  const int rows_used = p.G * p.P;
  if (rows_used < 128) {
    for (int i = tid; i < (128 - rows_used) * 8 * 2; i += THREADS) {
      const int half = i / ((128 - rows_used) * 8);
      const int rem = i % ((128 - rows_used) * 8);
      const int r = rows_used + rem / 8;
      const int ch = rem % 8;
      *reinterpret_cast<uint4*>(smem + half * (128 * 128) + r * 128 + ch * 16) = make_uint4(0, 0, 0, 0);
    }
    fence_proxy_async_smem();
  }
  const uint32_t* tile_mask = p.masks + ((long long)bg * p.n_ptiles + pt) * p.NBW;
  for (int w = tid; w < p.NBW; w += THREADS) words[w] = tile_mask[w];
  __syncthreads();

  // Block list: the tile's current block(s) first (descending), then every
  // historical block some row selects, descending.
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
        // keep only blocks below the lowest current block
        if (lo + 32 > cur_lo) bits &= (cur_lo - lo <= 0) ? 0u : ((cur_lo - lo >= 32) ? 0xffffffffu : ((1u << (cur_lo - lo)) - 1u));
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
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      mbar_expect_tx(&bars->q_full, (uint32_t)(p.G * p.P * 128 * 2));
      for (int hh = 0; hh < p.G; ++hh)
        for (int half = 0; half < 2; ++half)
          tma_load_3d(smem + half * (128 * 128) + hh * p.P * 128, &tmQ, &bars->q_full, half * 64, t0,
                      b * p.Hq + g * p.G + hh);
      int issued = 0;
      for (int j = 0; j < n; ++j) {
        const int st = j % NST;
        if (j >= NST && !mbar_wait(&bars->kv_empty[st], ((j / NST) - 1) & 1, status, p.wait_ns)) break;
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
      // Drain: wait for the copies still in flight before the CTA can exit.
      for (int j = max(0, issued - NST); j < issued; ++j) {
        mbar_wait_drain(&bars->k_full[j % NST], (j / NST) & 1);
        mbar_wait_drain(&bars->v_full[j % NST], (j / NST) & 1);
      }
      mbar_wait_drain(&bars->q_full, 0);
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc_s = make_idesc_bf16(128, 64, 0, 0);
      const uint32_t idesc_pv = make_idesc_bf16(128, D, 0, 1);
      bool ok = mbar_wait(&bars->q_full, 0, status, p.wait_ns);
      for (int j = 0; ok && j <= n; ++j) {
        if (j < n) {
          const int st = j % NST;
          const int sb = j & 1;
          ok = mbar_wait(&bars->k_full[st], (j / NST) & 1, status, p.wait_ns);
          // S buffer sb held S and then P of block j-2: free once that P V has completed.
          if (ok && j >= 2) ok = mbar_wait(&bars->pv_done[sb], ((j - 2) >> 1) & 1, status, p.wait_ns);
          if (!ok) break;
          tc_fence_after();
          const uint32_t kb = s_base + OFF_KV + st * STAGE_BYTES;
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks) {
            const uint32_t half = ks >> 2, koff = (ks & 3) * 32;
            const uint64_t a = make_sdesc(s_base + half * (128 * 128) + koff, 16, 1024);
            const uint64_t bd = make_sdesc(kb + half * KV_HALF + koff, 16, 1024);
            umma_ss(tmem + COL_S0 + 64 * sb, a, bd, idesc_s, ks > 0 ? 1u : 0u);
          }
          umma_commit(&bars->s_full[sb]);
        }
        if (j >= 1) {
          const int jj = j - 1;
          const int st = jj % NST;
          const int pb = jj & 1;
          ok = mbar_wait(&bars->p_full[pb], (jj >> 1) & 1, status, p.wait_ns);
          if (ok) ok = mbar_wait(&bars->v_full[st], (jj / NST) & 1, status, p.wait_ns);
          if (!ok) break;
          tc_fence_after();
          const uint32_t vb = s_base + OFF_KV + st * STAGE_BYTES + 2 * KV_HALF;
#pragma unroll
          for (int ks = 0; ks < 4; ++ks) {
            const uint64_t bd = make_sdesc(vb + ks * 2048, KV_HALF, 1024);
            umma_ts(tmem + COL_O, tmem + COL_S0 + 64 * pb + ks * 8, bd, idesc_pv, (jj > 0 || ks > 0) ? 1u : 0u);
          }
          umma_commit(&bars->pv_done[pb]);
          umma_commit(&bars->kv_empty[st]);
        }
      }
      // All issued MMAs complete before TMEM is released.
      umma_commit(&bars->fin);
      mbar_wait_drain(&bars->fin, 0);
    }
  } else {
    // ------------------------------------------------------------ softmax warps 0-3
    const int r = tid;   // row = TMEM lane
    const int hh = r / p.P;
    const int pp = r % p.P;
    const int t = t0 + pp;
    const bool valid = (r < rows_used) && (t < p.T);
    const int c_t = valid ? t / kBlock : -1;
    const long long grow = (long long)bg * p.T + (valid ? t : 0);
    const float tau_t = valid ? p.tau[grow] : INFINITY;
    const int tidx_t = valid ? p.tau_idx[grow] : -1;
    const float* gate_row = p.logG + grow * (long long)p.NB;
    const float grl = (valid && p.gate_lse) ? p.gate_lse[grow] : 0.f;   // log g = s - LSE(s) for raw scores
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    float m_used = -INFINITY;
    float l = 0.f;
    bool ok = true;
    float gate_next = 0.f;
    if (n > 0) {
      const int m0 = list[0];
      gate_next = (valid && m0 < c_t) ? __ldg(gate_row + m0) - grl : 0.f;
    }
    for (int j = 0; j < n; ++j) {
      const int m = list[j];
      const int sb = j & 1;
      const float gv = gate_next;
      if (j + 1 < n) {
        const int mn = list[j + 1];
        gate_next = (valid && mn < c_t) ? __ldg(gate_row + mn) - grl : 0.f;
      }
      // Row bias for this block: own block causal, selected historical gated, rest masked.
      bool masked = true;
      int lim = 63;
      float bias2 = 0.f;
      if (valid) {
        if (m == c_t) {
          masked = false;
          lim = t - m * kBlock;
        } else if (m < c_t && (gv > tau_t || (gv == tau_t && m <= tidx_t))) {
          masked = false;
          bias2 = gv * kLog2e;
        }
      }
      ok = warp_wait(&bars->s_full[sb], (j >> 1) & 1, status, p.wait_ns);
      if (!ok) break;
      tc_fence_after();
      uint32_t sr[2][32];
      tmem_ld32(tmem + lane_base + COL_S0 + 64 * sb, sr[0]);
      tmem_ld32(tmem + lane_base + COL_S0 + 64 * sb + 32, sr[1]);
      tmem_wait_ld();
      float x[64];
      float mx = -INFINITY;
#pragma unroll
      for (int k = 0; k < 64; ++k) {
        const float sv = __uint_as_float(sr[k >> 5][k & 31]);
        x[k] = (masked || k > lim) ? -INFINITY : fmaf(sv, p.scale_log2, bias2);
        mx = fmaxf(mx, x[k]);
      }
      const bool need = mx > m_used + RESCALE_THRESHOLD;   // false while mx == -inf
      const float m_new = need ? mx : m_used;
      // P buffer sb is free once the PV of block j-2 has completed.
      if (j >= 2) {
        ok = warp_wait(&bars->pv_done[sb], ((j - 2) >> 1) & 1, status, p.wait_ns);
        if (!ok) break;
      }
      const bool rescale_o = need && (m_used != -INFINITY) && (j > 0);
      if (__any_sync(0xffffffffu, rescale_o)) {
        // Every PV issued so far (through block j-1) must have landed in O.
        ok = warp_wait(&bars->pv_done[(j - 1) & 1], ((j - 1) >> 1) & 1, status, p.wait_ns);
        if (!ok) break;
        tc_fence_after();
        const float f = rescale_o ? ex2(m_used - m_new) : 1.f;
#pragma unroll 1
        for (int ch = 0; ch < D / 32; ++ch) {
          uint32_t o[32];
          tmem_ld32(tmem + lane_base + COL_O + 32 * ch, o);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * f);
          tmem_st32(tmem + lane_base + COL_O + 32 * ch, o);
        }
        tmem_wait_st();
      }
      if (need) {
        l = (m_used == -INFINITY) ? 0.f : l * ex2(m_used - m_new);
        m_used = m_new;
      }
      const float m_ref = (m_used == -INFINITY) ? 0.f : m_used;
      uint32_t pk[32];
      float rs = 0.f;
#pragma unroll
      for (int k = 0; k < 32; ++k) {
        const float a0 = ex2(x[2 * k] - m_ref);
        const float a1 = ex2(x[2 * k + 1] - m_ref);
        rs += a0 + a1;
        pk[k] = pack_bf16(a0, a1);
      }
      l += rs;
      tmem_st32(tmem + lane_base + COL_S0 + 64 * sb, pk);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->p_full[sb]);
    }
    // ---------------------------------------------------------- epilogue
    if (ok && n > 0) ok = warp_wait(&bars->pv_done[(n - 1) & 1], ((n - 1) >> 1) & 1, status, p.wait_ns);
    if (ok) {
      tc_fence_after();
      const float inv_l = (l > 0.f) ? 1.f / l : 0.f;
      const int h = g * p.G + hh;
      __nv_bfloat16* orow = p.O + (((long long)b * p.Hq + h) * p.T + t) * D;
#pragma unroll 1
      for (int ch = 0; ch < D / 32; ++ch) {
        uint32_t o[32];
        tmem_ld32(tmem + lane_base + COL_O + 32 * ch, o);
        tmem_wait_ld();
        if (valid) {
          uint32_t w[16];
#pragma unroll
          for (int k = 0; k < 16; ++k)
            w[k] = pack_bf16(__uint_as_float(o[2 * k]) * inv_l, __uint_as_float(o[2 * k + 1]) * inv_l);
          uint4* dst = reinterpret_cast<uint4*>(orow + 32 * ch);
#pragma unroll
          for (int k = 0; k < 4; ++k) dst[k] = make_uint4(w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
        }
      }
      if (valid) {
        const float m_ref = (m_used == -INFINITY) ? 0.f : m_used;
        p.LSE[((long long)b * p.Hq + h) * p.T + t] = (m_ref + __log2f(l)) * kLn2;
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

}  // namespace fwd

cudaError_t launch_fwd_tc(const TcProblem& pb, void* O, float* LSE, int32_t* status, uint32_t* masks,
                          cudaStream_t st) {
  const QTileShape qs = qtile_shape(pb.G, pb.T, pb.NB);
  cudaError_t e = launch_tile_union(pb.logG, pb.gate_lse, pb.tau, pb.tau_idx, masks, (long long)pb.B * pb.Hkv, pb.T,
                                    pb.NB, qs.P,
                                    qs.n_ptiles, qs.NBW, st);
  if (e != cudaSuccess) return e;
  CUtensorMap tq, tk, tv;
  if (!make_tmap_bf16_3d(&tq, pb.Q, pb.d, pb.T, (uint64_t)pb.B * pb.Hq, qs.P) ||
      !make_tmap_bf16_3d(&tk, pb.K, pb.d, pb.T, (uint64_t)pb.B * pb.Hkv, 64) ||
      !make_tmap_bf16_3d(&tv, pb.V, pb.d, pb.T, (uint64_t)pb.B * pb.Hkv, 64))
    return cudaErrorInvalidValue;
  fwd::Params prm;
  prm.logG = pb.logG;
  prm.gate_lse = pb.gate_lse;
  prm.tau = pb.tau;
  prm.tau_idx = pb.tau_idx;
  prm.masks = masks;
  prm.O = reinterpret_cast<__nv_bfloat16*>(O);
  prm.LSE = LSE;
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
  prm.wait_ns = wait_limit_ns();
  e = cudaFuncSetAttribute(fwd::sas_fwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, fwd::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  // All of L1 as shared memory, so that two CTAs fit on an SM.
  e = cudaFuncSetAttribute(fwd::sas_fwd_tc_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                           (int)cudaSharedmemCarveoutMaxShared);
  if (e != cudaSuccess) return e;
  const unsigned grid = (unsigned)((long long)pb.B * pb.Hkv * qs.n_ptiles);
  fwd::sas_fwd_tc_kernel<<<grid, fwd::THREADS, fwd::SMEM_BYTES, st>>>(tq, tk, tv, prm);
  count_launch();
  return cudaGetLastError();
}

}  // namespace sas
