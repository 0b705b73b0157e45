// fp32 SAS attention forward / backward on CUDA cores (fp32 storage and
// arithmetic throughout; used for the fp32 data type).
//
// SAS paper (arXiv 2609.13141) §4.3 eq. 9 and Appendix E: one CTA per (b, g,
// position t) with one warp per query head of the group. The warp walks only
// the row's attended blocks (its current block, causal, then every selected
// historical block), 32 keys at a time: lane j scores key j, the warp does the
// online softmax, and each lane accumulates D/32 output features.
#include "sas_common.cuh"
#include "sas_kernels.h"

namespace sas {
namespace simt {

struct Params {
  const float* Q;
  const float* K;
  const float* V;
  const float* O;
  const float* dO;
  const float* logG;       // log gates, or raw scores when gate_lse is set
  const float* gate_lse;   // null, or the LSE of each row's historical scores
  const float* tau;
  const int32_t* tau_idx;
  const float* LSE;
  const float* delta;
  float* outO;
  float* outLSE;
  float* dQ;
  float* dK;
  float* dV;
  float* dLogG;
  int B, Hq, Hkv, T, NB, G;
  float sm_scale;
};

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Next attended block after `m` for this row, in the order: current block c,
// then historical blocks 0..c-1 that pass the threshold. Returns -1 at the end.
__device__ __forceinline__ int next_block(int m, int c, const float* gate, float rl, float tau, int tidx) {
  int cand = (m == c) ? 0 : m + 1;
  if (m < 0) return c;
  for (; cand < c; ++cand) {
    const float v = gate[cand] - rl;
    if (v > tau || (v == tau && cand <= tidx)) return cand;
  }
  return -1;
}

template <int D>
__global__ void fwd_kernel(const Params p) {
  constexpr int NPL = D / 32;
  extern __shared__ float qs[];   // [G][D]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long row = blockIdx.x;   // (b * Hkv + g) * T + t
  const int t = (int)(row % p.T);
  const long long bg = row / p.T;
  const int b = (int)(bg / p.Hkv), g = (int)(bg % p.Hkv);
  const int h = g * p.G + warp;
  const long long qrow = ((long long)b * p.Hq + h) * p.T + t;
  float* q = qs + warp * D;
  for (int i = lane; i < D; i += 32) q[i] = p.Q[qrow * D + i];
  __syncwarp();
  const float* Kb = p.K + bg * (long long)p.T * D;
  const float* Vb = p.V + bg * (long long)p.T * D;
  const float* gate = p.logG + row * (long long)p.NB;
  const float rl = p.gate_lse ? p.gate_lse[row] : 0.f;   // raw scores: log g = s - LSE(s)
  const float tau = p.tau[row];
  const int tidx = p.tau_idx[row];
  const int c = t / kBlock;
  float mrun = -INFINITY, l = 0.f;
  float acc[NPL];
#pragma unroll
  for (int i = 0; i < NPL; ++i) acc[i] = 0.f;
  for (int m = next_block(-1, c, gate, rl, tau, tidx); m >= 0; m = next_block(m, c, gate, rl, tau, tidx)) {
    const float bias = (m == c) ? 0.f : gate[m] - rl;
    for (int ch = 0; ch < 2; ++ch) {
      const int key = m * kBlock + ch * 32 + lane;
      const bool ok = (m != c) || key <= t;
      float sc = -INFINITY;
      if (ok) {
        float dot = 0.f;
        const float* kr = Kb + (long long)key * D;
#pragma unroll 8
        for (int i = 0; i < D; ++i) dot = fmaf(q[i], kr[i], dot);
        sc = dot * p.sm_scale + bias;
      }
      const float cm = warp_max(sc);
      if (cm == -INFINITY) continue;
      const float mnew = fmaxf(mrun, cm);
      const float f = expf(mrun - mnew);   // 0 when mrun = -inf
      const float pr = ok ? expf(sc - mnew) : 0.f;
      l = l * f + warp_sum(pr);
#pragma unroll
      for (int i = 0; i < NPL; ++i) acc[i] *= f;
      for (int j = 0; j < 32; ++j) {
        const float pj = __shfl_sync(0xffffffffu, pr, j);
        if (pj != 0.f) {
          const float* vr = Vb + (long long)(m * kBlock + ch * 32 + j) * D;
#pragma unroll
          for (int i = 0; i < NPL; ++i) acc[i] = fmaf(pj, vr[lane + 32 * i], acc[i]);
        }
      }
      mrun = mnew;
    }
  }
  const float inv = 1.f / l;
#pragma unroll
  for (int i = 0; i < NPL; ++i) p.outO[qrow * D + lane + 32 * i] = acc[i] * inv;
  if (lane == 0) p.outLSE[qrow] = mrun + logf(l);
}

__global__ void delta_kernel_f32(const float* __restrict__ O, const float* __restrict__ dO, float* __restrict__ delta,
                                 long long rows, int D) {
  const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  float acc = 0.f;
  for (int i = lane; i < D; i += 32) acc = fmaf(O[row * D + i], dO[row * D + i], acc);
  acc = warp_sum(acc);
  if (lane == 0) delta[row] = acc;
}

template <int D>
__global__ void bwd_kernel(const Params p) {
  constexpr int NPL = D / 32;
  extern __shared__ float sh[];   // q [G][D], do [G][D], red [G]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long row = blockIdx.x;
  const int t = (int)(row % p.T);
  const long long bg = row / p.T;
  const int b = (int)(bg / p.Hkv), g = (int)(bg % p.Hkv);
  const int h = g * p.G + warp;
  const long long qrow = ((long long)b * p.Hq + h) * p.T + t;
  float* q = sh + warp * D;
  float* dov = sh + p.G * D + warp * D;
  float* red = sh + 2 * p.G * D;
  for (int i = lane; i < D; i += 32) {
    q[i] = p.Q[qrow * D + i];
    dov[i] = p.dO[qrow * D + i];
  }
  __syncwarp();
  const float* Kb = p.K + bg * (long long)p.T * D;
  const float* Vb = p.V + bg * (long long)p.T * D;
  float* dKb = p.dK + bg * (long long)p.T * D;
  float* dVb = p.dV + bg * (long long)p.T * D;
  const float* gate = p.logG + row * (long long)p.NB;
  const float rl = p.gate_lse ? p.gate_lse[row] : 0.f;   // raw scores: log g = s - LSE(s)
  const float tau = p.tau[row];
  const int tidx = p.tau_idx[row];
  const int c = t / kBlock;
  const float lse = p.LSE[qrow];
  const float dlt = p.delta[qrow];
  float dq[NPL];
#pragma unroll
  for (int i = 0; i < NPL; ++i) dq[i] = 0.f;
  for (int m = next_block(-1, c, gate, rl, tau, tidx); m >= 0; m = next_block(m, c, gate, rl, tau, tidx)) {
    const float bias = (m == c) ? 0.f : gate[m] - rl;
    float blk = 0.f;
    for (int ch = 0; ch < 2; ++ch) {
      const int key = m * kBlock + ch * 32 + lane;
      const bool ok = (m != c) || key <= t;
      float pr = 0.f, ds = 0.f;
      if (ok) {
        float dot = 0.f, dpv = 0.f;
        const float* kr = Kb + (long long)key * D;
        const float* vr = Vb + (long long)key * D;
#pragma unroll 8
        for (int i = 0; i < D; ++i) {
          dot = fmaf(q[i], kr[i], dot);
          dpv = fmaf(dov[i], vr[i], dpv);
        }
        pr = expf(dot * p.sm_scale + bias - lse);
        ds = pr * (dpv - dlt);
      }
      blk += warp_sum(ds);
      for (int j = 0; j < 32; ++j) {
        const float dsj = __shfl_sync(0xffffffffu, ds, j);
        const float pj = __shfl_sync(0xffffffffu, pr, j);
        if (pj == 0.f && dsj == 0.f) continue;
        const long long kj = (long long)(m * kBlock + ch * 32 + j) * D;
#pragma unroll
        for (int i = 0; i < NPL; ++i) {
          const int dd = lane + 32 * i;
          dq[i] = fmaf(dsj, Kb[kj + dd], dq[i]);
          atomicAdd(dKb + kj + dd, p.sm_scale * dsj * q[dd]);
          atomicAdd(dVb + kj + dd, pj * dov[dd]);
        }
      }
    }
    if (m != c) {
      if (lane == 0) red[warp] = blk;
      __syncthreads();
      if (threadIdx.x == 0) {
        float s = 0.f;
        for (int w = 0; w < p.G; ++w) s += red[w];
        p.dLogG[row * (long long)p.NB + m] = s;
      }
      __syncthreads();
    }
  }
#pragma unroll
  for (int i = 0; i < NPL; ++i) p.dQ[qrow * D + lane + 32 * i] = dq[i] * p.sm_scale;
}

Params make_params(const TcProblem& pb) {
  Params prm{};
  prm.Q = static_cast<const float*>(pb.Q);
  prm.K = static_cast<const float*>(pb.K);
  prm.V = static_cast<const float*>(pb.V);
  prm.O = static_cast<const float*>(pb.O);
  prm.dO = static_cast<const float*>(pb.dO);
  prm.logG = pb.logG;
  prm.gate_lse = pb.gate_lse;
  prm.tau = pb.tau;
  prm.tau_idx = pb.tau_idx;
  prm.LSE = pb.LSE;
  prm.B = pb.B;
  prm.Hq = pb.Hq;
  prm.Hkv = pb.Hkv;
  prm.T = pb.T;
  prm.NB = pb.NB;
  prm.G = pb.G;
  prm.sm_scale = pb.sm_scale;
  return prm;
}

}  // namespace simt

cudaError_t launch_fwd_simt(const TcProblem& pb, float* O, float* LSE, cudaStream_t st) {
  simt::Params prm = simt::make_params(pb);
  prm.outO = O;
  prm.outLSE = LSE;
  const unsigned grid = (unsigned)((long long)pb.B * pb.Hkv * pb.T);
  const size_t shm = (size_t)pb.G * pb.d * sizeof(float);
  if (pb.d == 128)
    simt::fwd_kernel<128><<<grid, 32 * pb.G, shm, st>>>(prm);
  else
    simt::fwd_kernel<64><<<grid, 32 * pb.G, shm, st>>>(prm);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_bwd_simt(const TcProblem& pb, float* dQ, float* dK, float* dV, float* dLogG, float* delta,
                            cudaStream_t st) {
  const size_t kv_bytes = (size_t)pb.B * pb.Hkv * pb.T * pb.d * sizeof(float);
  cudaError_t e;
  if ((e = cudaMemsetAsync(dK, 0, kv_bytes, st)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(dV, 0, kv_bytes, st)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(dLogG, 0, (size_t)pb.B * pb.Hkv * pb.T * pb.NB * sizeof(float), st)) != cudaSuccess)
    return e;
  const long long qrows = (long long)pb.B * pb.Hq * pb.T;
  simt::delta_kernel_f32<<<(unsigned)((qrows + 7) / 8), 256, 0, st>>>(static_cast<const float*>(pb.O),
                                                                     static_cast<const float*>(pb.dO), delta, qrows,
                                                                     pb.d);
  count_launch();
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  simt::Params prm = simt::make_params(pb);
  prm.delta = delta;
  prm.dQ = dQ;
  prm.dK = dK;
  prm.dV = dV;
  prm.dLogG = dLogG;
  const unsigned grid = (unsigned)((long long)pb.B * pb.Hkv * pb.T);
  const size_t shm = (size_t)(2 * pb.G * pb.d + pb.G) * sizeof(float);
  if (pb.d == 128)
    simt::bwd_kernel<128><<<grid, 32 * pb.G, shm, st>>>(prm);
  else
    simt::bwd_kernel<64><<<grid, 32 * pb.G, shm, st>>>(prm);
  count_launch();
  return cudaGetLastError();
}

}  // namespace sas
