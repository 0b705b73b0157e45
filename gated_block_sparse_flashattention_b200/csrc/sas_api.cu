// C ABI of the SAS library: argument validation, workspace layout and dispatch
// to the kernels. Declared in include/sas.h.
#include <atomic>
#include <cstdint>
#include <cstring>

#include "sas.h"
#include "sas_kernels.h"

namespace sas {

static std::atomic<uint64_t> g_launches{0};
void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

// 1 s unless sas_set_wait_limit_ns() changed it.
static std::atomic<uint64_t> g_wait_limit_ns{1000000000ull};
uint64_t wait_limit_ns() { return g_wait_limit_ns.load(std::memory_order_relaxed); }

QTileShape qtile_shape(int G, int T, int NB) {
  QTileShape s;
  s.P = (128 / G) & ~7;
  s.n_ptiles = s.P > 0 ? (T + s.P - 1) / s.P : 0;
  s.NBW = (NB + 31) / 32;
  return s;
}

namespace {

constexpr int kMaxNBTensorCore = 4096;   // block-list capacity of the tensor-core kernels
constexpr int kMaxQTiles = 8192;         // q-tile list capacity of the dK/dV kernel
constexpr size_t kStatusBytes = 256;

inline size_t align256(size_t x) { return (x + 255) / 256 * 256; }
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool aligned256(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 255u) == 0; }
inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }
inline int cuda_status(cudaError_t e) { return e == cudaSuccess ? SAS_OK : SAS_ERR_CUDA; }

// Shared shape checks of sas_fwd / sas_bwd.
int check_attention_shape(int B, int Hq, int Hkv, int T, int d, int block, int dtype) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || T <= 0 || d <= 0) return SAS_ERR_INVALID_ARG;
  if (block != 64) return SAS_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return SAS_ERR_INVALID_ARG;
  if (T % 64 != 0) return SAS_ERR_INVALID_ARG;
  if (dtype != SAS_DT_F32 && dtype != SAS_DT_BF16) return SAS_ERR_INVALID_ARG;
  const int G = Hq / Hkv;
  if (dtype == SAS_DT_F32) {
    if (d != 64 && d != 128) return SAS_ERR_UNSUPPORTED;
    if (G > 32) return SAS_ERR_UNSUPPORTED;
  } else {
    if (d != 128) return SAS_ERR_UNSUPPORTED;
    if (G > 16) return SAS_ERR_UNSUPPORTED;
    if (T / 64 > kMaxNBTensorCore) return SAS_ERR_UNSUPPORTED;
    if (qtile_shape(G, T, T / 64).n_ptiles > kMaxQTiles) return SAS_ERR_UNSUPPORTED;
  }
  if ((long long)B * Hq * T > (1ll << 31) - 1) return SAS_ERR_UNSUPPORTED;
  return SAS_OK;
}

size_t masks_bytes(int B, int Hkv, int T, int G) {
  const QTileShape qs = qtile_shape(G, T, T / 64);
  return align256((size_t)B * Hkv * qs.n_ptiles * qs.NBW * sizeof(uint32_t));
}

}  // namespace
}  // namespace sas

using namespace sas;

extern "C" {

const char* sas_status_string(int status) {
  switch (status) {
    case SAS_OK: return "SAS_OK";
    case SAS_ERR_INVALID_ARG: return "SAS_ERR_INVALID_ARG: invalid argument";
    case SAS_ERR_UNSUPPORTED: return "SAS_ERR_UNSUPPORTED: shape or dtype not supported by this build";
    case SAS_ERR_CUDA: return "SAS_ERR_CUDA: a CUDA runtime call failed";
    case SAS_ERR_TIMEOUT: return "SAS_ERR_TIMEOUT: a kernel's bounded wait expired";
    case SAS_ERR_WORKSPACE: return "SAS_ERR_WORKSPACE: workspace missing or too small";
    default: return "unknown sas_status";
  }
}

int sas_version(void) { return 100; }

uint64_t sas_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

uint64_t sas_set_wait_limit_ns(uint64_t ns) {
  const uint64_t v = ns == 0 ? 1000000000ull : ns;
  return g_wait_limit_ns.exchange(v, std::memory_order_relaxed);
}

int sas_gate_normalize(const float* s, float* logG, int B, int Hkv, int T, int NB, int block, void* stream) {
  if (!s || !logG || !aligned16(s) || !aligned16(logG) || s == logG) return SAS_ERR_INVALID_ARG;
  if (B <= 0 || Hkv <= 0 || T <= 0 || NB <= 0 || block != 64) return SAS_ERR_INVALID_ARG;
  if ((long long)NB * 64 < T) return SAS_ERR_INVALID_ARG;
  return cuda_status(launch_gate_normalize(s, logG, (long long)B * Hkv * T, T, NB, as_stream(stream)));
}

int sas_select_threshold(const float* logG, float* tau, int32_t* tau_idx, int32_t* sel, int B, int Hkv, int T,
                         int NB, int block, int K, void* stream) {
  if (!logG || !tau || !tau_idx || !aligned16(logG) || !aligned16(tau) || !aligned16(tau_idx))
    return SAS_ERR_INVALID_ARG;
  if (sel && !aligned16(sel)) return SAS_ERR_INVALID_ARG;
  if (B <= 0 || Hkv <= 0 || T <= 0 || NB <= 0 || block != 64 || K < 1) return SAS_ERR_INVALID_ARG;
  if ((long long)NB * 64 < T) return SAS_ERR_INVALID_ARG;
  return cuda_status(
      launch_select_threshold(logG, tau, tau_idx, sel, (long long)B * Hkv * T, T, NB, K - 1, as_stream(stream)));
}

int sas_gate_normalize_select(const float* s, float* logG, float* tau, int32_t* tau_idx, int32_t* sel, int B, int Hkv,
                              int T, int NB, int block, int K, void* stream) {
  if (!s || !logG || !tau || !tau_idx || s == logG) return SAS_ERR_INVALID_ARG;
  if (!aligned16(s) || !aligned16(logG) || !aligned16(tau) || !aligned16(tau_idx)) return SAS_ERR_INVALID_ARG;
  if (sel && !aligned16(sel)) return SAS_ERR_INVALID_ARG;
  if (B <= 0 || Hkv <= 0 || T <= 0 || NB <= 0 || block != 64 || K < 1) return SAS_ERR_INVALID_ARG;
  if ((long long)NB * 64 < T) return SAS_ERR_INVALID_ARG;
  return cuda_status(
      launch_normalize_select(s, logG, tau, tau_idx, sel, (long long)B * Hkv * T, T, NB, K - 1, as_stream(stream)));
}

int sas_gate_normalize_select_compact(const float* s, float* gate_lse, float* tau, int32_t* tau_idx, int32_t* sel,
                                      int B, int Hkv, int T, int NB, int block, int K, void* stream) {
  if (!s || !gate_lse || !tau || !tau_idx) return SAS_ERR_INVALID_ARG;
  if (!aligned16(s) || !aligned16(gate_lse) || !aligned16(tau) || !aligned16(tau_idx)) return SAS_ERR_INVALID_ARG;
  if (sel && !aligned16(sel)) return SAS_ERR_INVALID_ARG;
  if (B <= 0 || Hkv <= 0 || T <= 0 || NB <= 0 || block != 64 || K < 1) return SAS_ERR_INVALID_ARG;
  if ((long long)NB * 64 < T) return SAS_ERR_INVALID_ARG;
  if (NB > 1024) return SAS_ERR_UNSUPPORTED;   // rows are held in registers
  return cuda_status(launch_normalize_select_compact(s, gate_lse, tau, tau_idx, sel, (long long)B * Hkv * T, T, NB,
                                                     K - 1, as_stream(stream)));
}

int sas_gate_normalize_select_varlen(const float* s, float* logG, float* tau, int32_t* tau_idx, int32_t* sel, int B,
                                     int Hkv, int T, int NB, int block, int K, const int32_t* cu_seqlens,
                                     int n_docs, void* stream) {
  if (!s || !logG || !tau || !tau_idx || !cu_seqlens || s == logG) return SAS_ERR_INVALID_ARG;
  if (!aligned16(s) || !aligned16(logG) || !aligned16(tau) || !aligned16(tau_idx)) return SAS_ERR_INVALID_ARG;
  if (sel && !aligned16(sel)) return SAS_ERR_INVALID_ARG;
  if (B <= 0 || Hkv <= 0 || T <= 0 || NB <= 0 || block != 64 || K < 1) return SAS_ERR_INVALID_ARG;
  if ((long long)NB * 64 < T) return SAS_ERR_INVALID_ARG;
  if (n_docs < 1 || n_docs > kMaxDocs) return n_docs < 1 ? SAS_ERR_INVALID_ARG : SAS_ERR_UNSUPPORTED;
  if (NB > 1024) return SAS_ERR_UNSUPPORTED;   // rows are held in registers
  DocTable docs{};
  docs.n = n_docs;
  if (cu_seqlens[0] != 0 || cu_seqlens[n_docs] != T) return SAS_ERR_INVALID_ARG;
  for (int i = 0; i < n_docs; ++i) {
    if (cu_seqlens[i + 1] <= cu_seqlens[i] || cu_seqlens[i] % 64 != 0) return SAS_ERR_INVALID_ARG;
    docs.start_blk[i] = cu_seqlens[i] / 64;
  }
  return cuda_status(launch_normalize_select_varlen(s, logG, tau, tau_idx, sel, (long long)B * Hkv * T, T, NB, K - 1,
                                                    docs, as_stream(stream)));
}

int sas_select_noisy(const float* logG, const float* noise, float* logG_sel, float* tau, int32_t* tau_idx,
                     int32_t* sel, int B, int Hkv, int T, int NB, int block, int K, void* stream) {
  if (!logG || !noise || !logG_sel || !tau || !tau_idx) return SAS_ERR_INVALID_ARG;
  if (logG_sel == logG || logG_sel == noise) return SAS_ERR_INVALID_ARG;
  if (!aligned16(logG) || !aligned16(noise) || !aligned16(logG_sel) || !aligned16(tau) || !aligned16(tau_idx))
    return SAS_ERR_INVALID_ARG;
  if (sel && !aligned16(sel)) return SAS_ERR_INVALID_ARG;
  if (B <= 0 || Hkv <= 0 || T <= 0 || NB <= 0 || block != 64 || K < 1) return SAS_ERR_INVALID_ARG;
  if ((long long)NB * 64 < T) return SAS_ERR_INVALID_ARG;
  if (NB > 1024) return SAS_ERR_UNSUPPORTED;   // rows are held in registers
  return cuda_status(launch_select_noisy(logG, noise, logG_sel, tau, tau_idx, sel, (long long)B * Hkv * T, T, NB,
                                         K - 1, as_stream(stream)));
}

int sas_gate_grad(const float* logG, const float* gate_lse, const float* dLogG, float* ds, int B, int Hkv, int T, int NB,
                  int block, void* stream) {
  if (!logG || !dLogG || !ds || ds == logG || ds == dLogG) return SAS_ERR_INVALID_ARG;
  if (!aligned16(logG) || !aligned16(dLogG) || !aligned16(ds)) return SAS_ERR_INVALID_ARG;
  if (gate_lse && (!aligned16(gate_lse) || gate_lse == ds)) return SAS_ERR_INVALID_ARG;
  if (B <= 0 || Hkv <= 0 || T <= 0 || NB <= 0 || block != 64) return SAS_ERR_INVALID_ARG;
  if ((long long)NB * 64 < T) return SAS_ERR_INVALID_ARG;
  return cuda_status(launch_gate_grad(logG, gate_lse, dLogG, ds, (long long)B * Hkv * T, T, NB, as_stream(stream)));
}

int sas_fwd_workspace_size(int B, int Hq, int Hkv, int T, int d, int block, int K, int dtype, size_t* bytes) {
  if (!bytes || K < 1) return SAS_ERR_INVALID_ARG;
  const int st = check_attention_shape(B, Hq, Hkv, T, d, block, dtype);
  if (st != SAS_OK) return st;
  size_t n = kStatusBytes;
  if (dtype == SAS_DT_BF16)
    n += fwd_gather_applies(B, Hq, Hkv, T, K) ? fwd_gather_workspace_bytes(B, Hq, Hkv, T, K)
                                              : masks_bytes(B, Hkv, T, Hq / Hkv);
  *bytes = n;
  return SAS_OK;
}

int sas_bwd_workspace_size(int B, int Hq, int Hkv, int T, int d, int block, int K, int dtype, size_t* bytes) {
  if (!bytes || K < 1) return SAS_ERR_INVALID_ARG;
  const int st = check_attention_shape(B, Hq, Hkv, T, d, block, dtype);
  if (st != SAS_OK) return st;
  size_t n = kStatusBytes + align256((size_t)B * Hq * T * sizeof(float));   // Delta
  if (dtype == SAS_DT_BF16) n += bwd_gather_workspace_bytes(B, Hq, Hkv, T, K);
  *bytes = n;
  return SAS_OK;
}

int sas_decode_workspace_size(int B, int Hq, int Hkv, int Lmax, int d, int block, int K, size_t* bytes) {
  if (!bytes || B <= 0 || Hq <= 0 || Hkv <= 0 || Lmax <= 0 || block != 64 || K < 1 || Hq % Hkv != 0)
    return SAS_ERR_INVALID_ARG;
  if (d != 128 || K > 64 || Hq / Hkv > 16) return SAS_ERR_UNSUPPORTED;
  *bytes = decode_workspace_bytes(B, Hq, Hkv, K);
  return SAS_OK;
}

int sas_fwd(const void* Q, const void* K, const void* V, int dtype, const float* logG, const float* gate_lse,
            const float* tau, const int32_t* tau_idx, const int32_t* sel, void* O, float* LSE, int B, int Hq, int Hkv,
            int T, int d, int block, int Kbudget, float sm_scale, void* ws, size_t ws_bytes, void* stream) {
  const void* ptrs[] = {Q, K, V, logG, tau, tau_idx, O, LSE};
  for (const void* p : ptrs)
    if (!p || !aligned16(p)) return SAS_ERR_INVALID_ARG;
  if ((gate_lse && !aligned16(gate_lse)) || (sel && !aligned16(sel))) return SAS_ERR_INVALID_ARG;
  int st = check_attention_shape(B, Hq, Hkv, T, d, block, dtype);
  if (st != SAS_OK) return st;
  if (!(sm_scale > 0.f) || Kbudget < 1) return SAS_ERR_INVALID_ARG;
  size_t need = 0;
  sas_fwd_workspace_size(B, Hq, Hkv, T, d, block, Kbudget, dtype, &need);
  if (!ws || !aligned256(ws) || ws_bytes < need) return SAS_ERR_WORKSPACE;
  TcProblem pb{};
  pb.B = B;
  pb.Hq = Hq;
  pb.Hkv = Hkv;
  pb.T = T;
  pb.d = d;
  pb.NB = T / 64;
  pb.G = Hq / Hkv;
  pb.sm_scale = sm_scale;
  pb.Q = Q;
  pb.K = K;
  pb.V = V;
  pb.logG = logG;
  pb.gate_lse = gate_lse;
  pb.tau = tau;
  pb.tau_idx = tau_idx;
  pb.sel = sel;
  cudaStream_t s = as_stream(stream);
  uint8_t* w = static_cast<uint8_t*>(ws);
  if (dtype == SAS_DT_F32) return cuda_status(launch_fwd_simt(pb, static_cast<float*>(O), LSE, s));
  if (fwd_gather_applies(B, Hq, Hkv, T, Kbudget))
    return cuda_status(launch_fwd_gather(pb, Kbudget, O, LSE, reinterpret_cast<int32_t*>(w), w + kStatusBytes, s));
  return cuda_status(launch_fwd_tc(pb, O, LSE, reinterpret_cast<int32_t*>(w),
                                   reinterpret_cast<uint32_t*>(w + kStatusBytes), s));
}

int sas_bwd(const void* Q, const void* K, const void* V, const void* O, const void* dO, int dtype,
            const float* logG, const float* gate_lse, const float* tau, const int32_t* tau_idx, const int32_t* sel,
            const float* LSE, void* dQ, void* dK, void* dV, float* dLogG, int B, int Hq, int Hkv, int T, int d,
            int block, int Kbudget, float sm_scale, void* ws, size_t ws_bytes, void* stream) {
  const void* ptrs[] = {Q, K, V, O, dO, logG, tau, tau_idx, LSE, dQ, dK, dV, dLogG};
  for (const void* p : ptrs)
    if (!p || !aligned16(p)) return SAS_ERR_INVALID_ARG;
  if ((gate_lse && !aligned16(gate_lse)) || (sel && !aligned16(sel))) return SAS_ERR_INVALID_ARG;
  int st = check_attention_shape(B, Hq, Hkv, T, d, block, dtype);
  if (st != SAS_OK) return st;
  if (!(sm_scale > 0.f)) return SAS_ERR_INVALID_ARG;
  size_t need = 0;
  if (Kbudget < 1) return SAS_ERR_INVALID_ARG;
  sas_bwd_workspace_size(B, Hq, Hkv, T, d, block, Kbudget, dtype, &need);
  if (!ws || !aligned256(ws) || ws_bytes < need) return SAS_ERR_WORKSPACE;
  TcProblem pb{};
  pb.B = B;
  pb.Hq = Hq;
  pb.Hkv = Hkv;
  pb.T = T;
  pb.d = d;
  pb.NB = T / 64;
  pb.G = Hq / Hkv;
  pb.sm_scale = sm_scale;
  pb.Q = Q;
  pb.K = K;
  pb.V = V;
  pb.O = O;
  pb.dO = dO;
  pb.logG = logG;
  pb.gate_lse = gate_lse;
  pb.tau = tau;
  pb.tau_idx = tau_idx;
  pb.sel = sel;
  pb.LSE = LSE;
  cudaStream_t s = as_stream(stream);
  uint8_t* w = static_cast<uint8_t*>(ws);
  float* delta = reinterpret_cast<float*>(w + kStatusBytes);
  if (dtype == SAS_DT_F32)
    return cuda_status(launch_bwd_simt(pb, static_cast<float*>(dQ), static_cast<float*>(dK), static_cast<float*>(dV),
                                       dLogG, delta, s));
  uint8_t* scratch = w + kStatusBytes + align256((size_t)B * Hq * T * sizeof(float));
  return cuda_status(
      launch_bwd_gather(pb, Kbudget, dQ, dK, dV, dLogG, reinterpret_cast<int32_t*>(w), delta, scratch, s));
}

int sas_decode_fwd(const void* q, const void* Kc, const void* Vc, int dtype, const int32_t* seqlen, const float* s,
                   int K, int apply_log_gate, void* o, int32_t* sel_out, int B, int Hq, int Hkv, int Lmax, int NBmax,
                   int d, int block, float sm_scale, void* ws, size_t ws_bytes, void* stream) {
  const void* ptrs[] = {q, Kc, Vc, seqlen, s, o};
  for (const void* p : ptrs)
    if (!p || !aligned16(p)) return SAS_ERR_INVALID_ARG;
  if (sel_out && !aligned16(sel_out)) return SAS_ERR_INVALID_ARG;
  if (dtype != SAS_DT_F32 && dtype != SAS_DT_BF16) return SAS_ERR_INVALID_ARG;
  if ((long long)NBmax * 64 < Lmax || !(sm_scale > 0.f)) return SAS_ERR_INVALID_ARG;
  size_t need = 0;
  int st = sas_decode_workspace_size(B, Hq, Hkv, Lmax, d, block, K, &need);
  if (st != SAS_OK) return st;
  if (!ws || !aligned256(ws) || ws_bytes < need) return SAS_ERR_WORKSPACE;
  DecodeProblem pb{};
  pb.B = B;
  pb.Hq = Hq;
  pb.Hkv = Hkv;
  pb.Lmax = Lmax;
  pb.NBmax = NBmax;
  pb.d = d;
  pb.K = K;
  pb.apply_log_gate = apply_log_gate ? 1 : 0;
  pb.dtype = dtype;
  pb.sm_scale = sm_scale;
  pb.q = q;
  pb.Kc = Kc;
  pb.Vc = Vc;
  pb.seqlen = seqlen;
  pb.s = s;
  pb.o = o;
  pb.sel_out = sel_out;
  return cuda_status(launch_decode(pb, ws, as_stream(stream)));
}

int sas_decode_fwd_paged(const void* q, const void* Kp, const void* Vp, int dtype, const int32_t* page_table,
                         int max_pages, int num_pages, const int32_t* seqlen, const float* s, int K, int apply_log_gate,
                         void* o, int32_t* sel_out, int B, int Hq, int Hkv, int NBmax, int d, int block,
                         float sm_scale, void* ws, size_t ws_bytes, void* stream) {
  const void* ptrs[] = {q, Kp, Vp, page_table, seqlen, s, o};
  for (const void* p : ptrs)
    if (!p || !aligned16(p)) return SAS_ERR_INVALID_ARG;
  if (sel_out && !aligned16(sel_out)) return SAS_ERR_INVALID_ARG;
  if (dtype != SAS_DT_F32 && dtype != SAS_DT_BF16) return SAS_ERR_INVALID_ARG;
  if (dtype != SAS_DT_BF16) return SAS_ERR_UNSUPPORTED;   // the paged path is the tensor-core kernel
  if (max_pages < 1 || num_pages < 1 || Hkv <= 0) return SAS_ERR_INVALID_ARG;
  if ((long long)max_pages * 64 > INT32_MAX || (long long)num_pages * Hkv > INT32_MAX) return SAS_ERR_INVALID_ARG;
  if (NBmax < max_pages || !(sm_scale > 0.f)) return SAS_ERR_INVALID_ARG;
  const int Lmax = max_pages * 64;
  size_t need = 0;
  int st = sas_decode_workspace_size(B, Hq, Hkv, Lmax, d, block, K, &need);
  if (st != SAS_OK) return st;
  if (!ws || !aligned256(ws) || ws_bytes < need) return SAS_ERR_WORKSPACE;
  DecodeProblem pb{};
  pb.B = B;
  pb.Hq = Hq;
  pb.Hkv = Hkv;
  pb.Lmax = Lmax;
  pb.NBmax = NBmax;
  pb.d = d;
  pb.K = K;
  pb.apply_log_gate = apply_log_gate ? 1 : 0;
  pb.dtype = dtype;
  pb.sm_scale = sm_scale;
  pb.q = q;
  pb.Kc = Kp;
  pb.Vc = Vp;
  pb.seqlen = seqlen;
  pb.s = s;
  pb.o = o;
  pb.sel_out = sel_out;
  pb.page_table = page_table;
  pb.max_pages = max_pages;
  pb.num_pages = num_pages;
  return cuda_status(launch_decode(pb, ws, as_stream(stream)));
}

int sas_decode_fwd_static(const void* q, const void* Kc, const void* Vc, int dtype, const int32_t* seqlen,
                          const float* s, int K, int apply_log_gate, void* o, int32_t* sel_out, int B, int Hq,
                          int Hkv, int Lmax, int NBmax, int d, int block, float sm_scale, void* stream) {
  const void* ptrs[] = {q, Kc, Vc, seqlen, s, o};
  for (const void* p : ptrs)
    if (!p || !aligned16(p)) return SAS_ERR_INVALID_ARG;
  if (sel_out && !aligned16(sel_out)) return SAS_ERR_INVALID_ARG;
  if (dtype != SAS_DT_F32 && dtype != SAS_DT_BF16) return SAS_ERR_INVALID_ARG;
  if ((long long)NBmax * 64 < Lmax || !(sm_scale > 0.f)) return SAS_ERR_INVALID_ARG;
  size_t need = 0;
  int st = sas_decode_workspace_size(B, Hq, Hkv, Lmax, d, block, K, &need);
  if (st != SAS_OK) return st;
  if (need > decode_static_scratch_limit()) return SAS_ERR_WORKSPACE;   // beyond the built-in scratch
  DecodeProblem pb{};
  pb.B = B;
  pb.Hq = Hq;
  pb.Hkv = Hkv;
  pb.Lmax = Lmax;
  pb.NBmax = NBmax;
  pb.d = d;
  pb.K = K;
  pb.apply_log_gate = apply_log_gate ? 1 : 0;
  pb.dtype = dtype;
  pb.sm_scale = sm_scale;
  pb.q = q;
  pb.Kc = Kc;
  pb.Vc = Vc;
  pb.seqlen = seqlen;
  pb.s = s;
  pb.o = o;
  pb.sel_out = sel_out;
  return cuda_status(launch_decode_static(pb, as_stream(stream)));
}

int sas_decode_static_status(void* stream, int32_t* status_out) {
  if (!status_out) return SAS_ERR_INVALID_ARG;
  int32_t v = 0;
  if (decode_static_status(as_stream(stream), &v) != cudaSuccess) return SAS_ERR_CUDA;
  *status_out = v;
  return v == 0 ? SAS_OK : SAS_ERR_TIMEOUT;
}

int sas_device_status(const void* ws, void* stream, int32_t* status_out) {
  if (!ws || !status_out) return SAS_ERR_INVALID_ARG;
  cudaError_t e = cudaStreamSynchronize(as_stream(stream));
  if (e != cudaSuccess) return SAS_ERR_CUDA;
  int32_t v = 0;
  e = cudaMemcpy(&v, ws, sizeof(v), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return SAS_ERR_CUDA;
  *status_out = v;
  return v == 0 ? SAS_OK : SAS_ERR_TIMEOUT;
}

int sas_device_status_clear(void* ws, void* stream) {
  if (!ws) return SAS_ERR_INVALID_ARG;
  return cuda_status(cudaMemsetAsync(ws, 0, sizeof(int32_t), as_stream(stream)));
}

}  // extern "C"
