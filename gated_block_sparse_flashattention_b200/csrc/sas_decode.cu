// SAS sparse decode step (memory-bound).
//
// SAS paper (arXiv 2609.13141) §4.3 Algorithm 2 (Top-K on the selector scores,
// then ungated attention over the current block and the selected blocks) and
// §5.1 "Inference implementation" (per-KV-group selection, GQA, gathering only
// the selected KV blocks).
//
// Grid: (b, g) x split. Every CTA recomputes the group's Top-(K-1) selection
// with one warp (radix select over the 2 KiB score row), then copies its share
// of the attended blocks (BPC blocks of 64 keys) from the KV cache into shared
// memory with one bulk async copy per block (untiled TMA), scores the G query
// heads of the group against them on CUDA cores, and writes an fp32 partial
// (row max, row sum, unnormalised output). The last CTA of a (b, g) to finish
// (atomic ticket) merges the partials into o.
#include <mutex>

#include "sas_common.cuh"
#include "sas_kernels.h"

namespace sas {
namespace decode {

constexpr int THREADS = 128;
constexpr int D = 128;
constexpr int BPC = 2;          // attended blocks per CTA

struct Params {
  const void* q;
  const void* Kc;
  const void* Vc;
  const int32_t* seqlen;
  const float* s;
  void* o;
  int32_t* sel_out;
  int32_t* status;     // device status word (first word of the workspace)
  int32_t* counters;   // [B*Hkv]
  float* part_ml;      // [B*Hkv][nsplit][G][2]
  float* part_o;       // [B*Hkv][nsplit][G][D]
  int B, Hq, Hkv, Lmax, NBmax, K, apply_log_gate, G, nsplit;
  float sm_scale;
};

__device__ __forceinline__ void bulk_copy_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

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

template <typename T>
__global__ void __launch_bounds__(THREADS) decode_kernel(const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  constexpr uint32_t BLK_BYTES = 64 * D * sizeof(T);
  T* kv = reinterpret_cast<T*>(smem);                                   // [BPC][2][64][D]
  float* qf = reinterpret_cast<float*>(smem + BPC * 2 * BLK_BYTES);      // [G][D]
  float* sc = qf + p.G * D;                                             // [G][BPC*64]
  uint32_t* hist = reinterpret_cast<uint32_t*>(sc + p.G * BPC * 64);     // [256]
  int* blk = reinterpret_cast<int*>(hist + 256);                        // [BPC] attended blocks of this CTA
  float* misc = reinterpret_cast<float*>(blk + BPC);                    // [0] = log-gate LSE
  uint64_t* bar = reinterpret_cast<uint64_t*>(misc + 4);
  int* last_flag = reinterpret_cast<int*>(bar + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bg = blockIdx.x / p.nsplit;
  const int split = blockIdx.x % p.nsplit;
  const int b = bg / p.Hkv, g = bg % p.Hkv;
  const int L = p.seqlen[b];
  const int c = (L - 1) / kBlock;
  const int H = p.K - 1;
  const float* srow = p.s + (long long)bg * p.NBmax;

  if (tid == 0) {
    mbar_init(bar, 1);
    fence_barrier_init();
  }
  if (warp == 0) {
    // ---- selection: attended list = [c, selected blocks ascending]
    float tauv = INFINITY;
    int tidx = -1;
    if (min(c, H) > 0) {
      if (c <= H) {
        tauv = -INFINITY;
        tidx = c - 1;
      } else {
        int take_eq = 0;
        const uint32_t tkey = warp_radix_select(srow, c, H, hist, &take_eq);
        tauv = key_float(tkey);
        int run = 0;
        for (int base = 0; base < c; base += 32) {
          const int m = base + lane;
          const bool eq = (m < c) && (float_key(srow[m]) == tkey);
          const uint32_t bal = __ballot_sync(0xffffffffu, eq);
          const int cnt = __popc(bal);
          if (run + cnt >= take_eq) {
            uint32_t bb = bal;
            for (int k = 1; k < take_eq - run; ++k) bb &= bb - 1u;
            tidx = base + __ffs(bb) - 1;
            break;
          }
          run += cnt;
        }
      }
    }
    // Walk the selected blocks in ascending order; list position 0 is block c.
    // mode 0: nothing selected, 1: every historical block, 2: threshold (tauv, tidx).
    const int mode = (min(c, H) == 0) ? 0 : (c <= H ? 1 : 2);
    const uint32_t tk = float_key(tauv);
    int pos = 1;
    int32_t* so = (p.sel_out && split == 0) ? p.sel_out + (long long)bg * H : nullptr;
    if (lane < BPC) blk[lane] = -1;
    __syncwarp();
    if (split == 0 && lane == 0) blk[0] = c;
    const int want_lo = split * BPC, want_hi = want_lo + BPC;
    for (int base = 0; mode != 0 && base < c && (pos < want_hi || so); base += 32) {
      const int m = base + lane;
      bool take = false;
      if (m < c) {
        if (mode == 1) {
          take = true;
        } else {
          const uint32_t k = float_key(srow[m]);
          take = (k > tk) || (k == tk && m <= tidx);
        }
      }
      const uint32_t bal = __ballot_sync(0xffffffffu, take);
      if (take) {
        const int lp = pos + __popc(bal & ((1u << lane) - 1u));
        if (lp >= want_lo && lp < want_hi) blk[lp - want_lo] = m;
        if (so) so[lp - 1] = m;
      }
      pos += __popc(bal);
    }
    if (so)
      for (int k = pos - 1 + lane; k < H; k += 32) so[k] = -1;
    if (p.apply_log_gate && c > 0) {
      float mx = -INFINITY;
      for (int m = lane; m < c; m += 32) mx = fmaxf(mx, srow[m]);
#pragma unroll
      for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      float sum = 0.f;
      for (int m = lane; m < c; m += 32) sum += expf(srow[m] - mx);
#pragma unroll
      for (int o = 16; o; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      if (lane == 0) misc[0] = mx + logf(sum);
    }
    __syncwarp();
    if (lane == 0) {
      // Issue the bulk copies of this CTA's blocks.
      uint32_t bytes = 0;
      for (int k = 0; k < BPC; ++k) {
        const int m = blk[k];
        if (m < 0) continue;
        const int rows = min(kBlock, p.Lmax - m * kBlock);
        bytes += 2u * rows * D * sizeof(T);
      }
      mbar_expect_tx(bar, bytes);
      for (int k = 0; k < BPC; ++k) {
        const int m = blk[k];
        if (m < 0) continue;
        const int rows = min(kBlock, p.Lmax - m * kBlock);
        const long long off = ((long long)bg * p.Lmax + (long long)m * kBlock) * D;
        bulk_copy_g2s(kv + (2 * k) * 64 * D, static_cast<const T*>(p.Kc) + off, rows * D * sizeof(T), bar);
        bulk_copy_g2s(kv + (2 * k + 1) * 64 * D, static_cast<const T*>(p.Vc) + off, rows * D * sizeof(T), bar);
      }
    }
  } else {
    // ---- q of the group's heads into shared memory (fp32)
    const T* qg = static_cast<const T*>(p.q) + ((long long)b * p.Hq + g * p.G) * D;
    for (int i = tid - 32; i < p.G * D; i += THREADS - 32) qf[i] = to_f<T>(qg[i]);
  }
  __syncthreads();
  const bool have = blk[0] >= 0;
  bool ok = true;
  if (have) ok = mbar_wait(bar, 0, p.status);
  const float lse_gate = (p.apply_log_gate && c > 0) ? misc[0] : 0.f;

  // ---- scores: sc[h][k*64 + key], masked keys -inf
  const int nkeys = BPC * 64;
  for (int idx = tid; idx < p.G * nkeys; idx += THREADS) {
    const int h = idx / nkeys, kk = idx % nkeys;
    const int k = kk / 64, key = kk % 64;
    const int m = blk[k];
    float v = -INFINITY;
    if (ok && m >= 0 && (m != c || m * kBlock + key <= L - 1)) {
      const T* kr = kv + (2 * k) * 64 * D + key * D;
      const float* qh = qf + h * D;
      float dot = 0.f;
#pragma unroll 4
      for (int i0 = 0; i0 < D; i0 += 8) {
        const int i = (i0 + 8 * (key & 15)) & (D - 1);   // rotate the start to spread shared-memory banks
#pragma unroll
        for (int e = 0; e < 8; ++e) dot = fmaf(qh[i + e], to_f<T>(kr[i + e]), dot);
      }
      v = dot * p.sm_scale;
      if (p.apply_log_gate && m != c) v += srow[m] - lse_gate;
    }
    sc[h * nkeys + kk] = v;
  }
  __syncthreads();
  // ---- per head: max and sum over this CTA's keys; p = exp(sc - max)
  for (int h = warp; h < p.G; h += THREADS / 32) {
    float mx = -INFINITY;
    for (int kk = lane; kk < nkeys; kk += 32) mx = fmaxf(mx, sc[h * nkeys + kk]);
#pragma unroll
    for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float sum = 0.f;
    for (int kk = lane; kk < nkeys; kk += 32) {
      const float e = (mx == -INFINITY) ? 0.f : expf(sc[h * nkeys + kk] - mx);
      sc[h * nkeys + kk] = e;
      sum += e;
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    if (lane == 0) {
      float* dst = p.part_ml + (((long long)bg * p.nsplit + split) * p.G + h) * 2;
      dst[0] = mx;
      dst[1] = sum;
    }
  }
  __syncthreads();
  // ---- partial output: thread = feature dd
  {
    const int dd = tid;
    for (int h = 0; h < p.G; ++h) {
      float acc = 0.f;
      for (int k = 0; k < BPC; ++k) {
        const int m = blk[k];
        if (m < 0) continue;
        // Only keys that exist in the cache were copied; rows past them are stale.
        const int nk = (m == c) ? (L - m * kBlock) : kBlock;
        const T* vb = kv + (2 * k + 1) * 64 * D;
        const float* ph = sc + h * nkeys + k * 64;
#pragma unroll 8
        for (int key = 0; key < nk; ++key) acc = fmaf(ph[key], to_f<T>(vb[key * D + dd]), acc);
      }
      p.part_o[(((long long)bg * p.nsplit + split) * p.G + h) * D + dd] = acc;
    }
  }
  // ---- the last CTA of this (b, g) merges the partials
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const int ticket = atomicAdd(p.counters + bg, 1);
    *last_flag = (ticket == p.nsplit - 1);
  }
  __syncthreads();
  if (*last_flag) {
    __threadfence();
    const int dd = tid;
    for (int h = 0; h < p.G; ++h) {
      const float* ml0 = p.part_ml + ((long long)bg * p.nsplit * p.G + h) * 2;
      float M = -INFINITY;
      for (int sp = 0; sp < p.nsplit; ++sp) M = fmaxf(M, __ldcg(ml0 + (long long)sp * p.G * 2));
      float num = 0.f, den = 0.f;
      for (int sp = 0; sp < p.nsplit; ++sp) {
        const float m_s = __ldcg(ml0 + (long long)sp * p.G * 2);
        if (m_s == -INFINITY) continue;
        const float w = expf(m_s - M);
        den += w * __ldcg(ml0 + (long long)sp * p.G * 2 + 1);
        num += w * __ldcg(p.part_o + (((long long)bg * p.nsplit + sp) * p.G + h) * D + dd);
      }
      const float out = num / den;
      const long long oi = ((long long)b * p.Hq + g * p.G + h) * D + dd;
      if constexpr (sizeof(T) == 2)
        static_cast<__nv_bfloat16*>(p.o)[oi] = __float2bfloat16_rn(out);
      else
        static_cast<float*>(p.o)[oi] = out;
    }
    if (tid == 0) p.counters[bg] = 0;   // ready for the next call
  }
}

}  // namespace decode

size_t decode_workspace_bytes(int B, int Hq, int Hkv, int K) {
  const int G = Hq / Hkv;
  const int nsplit = (K + decode::BPC - 1) / decode::BPC;
  const size_t n_bg = (size_t)B * Hkv;
  size_t bytes = 256;                                       // status word (first 4 bytes) + pad
  bytes += ((n_bg + 1) * sizeof(int32_t) + 255) / 256 * 256;   // tickets (+ a status slot)
  bytes += (n_bg * nsplit * G * 2 * sizeof(float) + 255) / 256 * 256;
  bytes += n_bg * nsplit * G * decode::D * sizeof(float);
  return bytes;
}

cudaError_t launch_decode(const DecodeProblem& pb, void* ws, cudaStream_t st) {
  using namespace decode;
  const int G = pb.Hq / pb.Hkv;
  const int nsplit = (pb.K + BPC - 1) / BPC;
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
  prm.counters = reinterpret_cast<int32_t*>(w + off);
  const size_t cnt_bytes = ((n_bg + 1) * sizeof(int32_t) + 255) / 256 * 256;
  off += cnt_bytes;
  prm.part_ml = reinterpret_cast<float*>(w + off);
  off += (n_bg * nsplit * G * 2 * sizeof(float) + 255) / 256 * 256;
  prm.part_o = reinterpret_cast<float*>(w + off);
  prm.B = pb.B;
  prm.Hq = pb.Hq;
  prm.Hkv = pb.Hkv;
  prm.Lmax = pb.Lmax;
  prm.NBmax = pb.NBmax;
  prm.K = pb.K;
  prm.apply_log_gate = pb.apply_log_gate;
  prm.G = G;
  prm.nsplit = nsplit;
  prm.sm_scale = pb.sm_scale;
  // Tickets start at zero on every call.
  cudaError_t e = cudaMemsetAsync(prm.counters, 0, n_bg * sizeof(int32_t), st);
  if (e != cudaSuccess) return e;
  const unsigned grid = (unsigned)(n_bg * nsplit);
  if (pb.dtype == 1) {
    const size_t shm = BPC * 2 * 64 * D * 2 + (size_t)G * D * 4 + (size_t)G * BPC * 64 * 4 + 256 * 4 + 64 + 128;
    e = cudaFuncSetAttribute(decode_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)shm);
    if (e != cudaSuccess) return e;
    decode_kernel<__nv_bfloat16><<<grid, THREADS, shm, st>>>(prm);
  } else {
    const size_t shm = BPC * 2 * 64 * D * 4 + (size_t)G * D * 4 + (size_t)G * BPC * 64 * 4 + 256 * 4 + 64 + 128;
    e = cudaFuncSetAttribute(decode_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)shm);
    if (e != cudaSuccess) return e;
    decode_kernel<float><<<grid, THREADS, shm, st>>>(prm);
  }
  count_launch();
  return cudaGetLastError();
}

}  // namespace sas

// ---------------------------------------------------------------------------
// Allocation-free variant of the decode step.
//
// Its scratch (status word, per-(b, g) tickets, split partials) lives in one
// file-scope device array instead of a caller workspace. Every GPU that loads
// the library keeps this array until the process exits, and every call on a
// device shares it, so calls that overlap on the GPU race on it.
// ---------------------------------------------------------------------------
namespace sas {
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
