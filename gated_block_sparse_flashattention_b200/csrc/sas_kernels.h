// Host-side declarations of the kernel launchers (internal to the library).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace sas {

// Counts one kernel launch (reported by sas_launch_count()).
void count_launch();
// Limit of one bounded wait inside the kernels that take it as a parameter
// (nanoseconds; sas_set_wait_limit_ns).
uint64_t wait_limit_ns();

cudaError_t launch_gate_normalize(const float* s, float* logG, long long rows, int T, int NB, cudaStream_t st);
cudaError_t launch_select_threshold(const float* logG, float* tau, int32_t* tau_idx, int32_t* sel, long long rows,
                                    int T, int NB, int H, cudaStream_t st);
cudaError_t launch_normalize_select(const float* s, float* logG, float* tau, int32_t* tau_idx, int32_t* sel,
                                    long long rows, int T, int NB, int H, cudaStream_t st);
// Document table of a packed sequence: the first block of each document.
constexpr int kMaxDocs = 256;
struct DocTable {
  int n;
  int start_blk[kMaxDocs];
};
cudaError_t launch_normalize_select_varlen(const float* s, float* logG, float* tau, int32_t* tau_idx, int32_t* sel,
                                           long long rows, int T, int NB, int H, const DocTable& docs,
                                           cudaStream_t st);
cudaError_t launch_select_noisy(const float* logG, const float* noise, float* logG_sel, float* tau, int32_t* tau_idx,
                                int32_t* sel, long long rows, int T, int NB, int H, cudaStream_t st);
cudaError_t launch_gate_grad(const float* logG, const float* gate_lse, const float* dLogG, float* ds, long long rows,
                             int T, int NB, cudaStream_t st);
cudaError_t launch_tile_union(const float* logG, const float* gate_lse, const float* tau, const int32_t* tau_idx,
                              uint32_t* masks, long long n_bg, int T, int NB, int P, int n_ptiles, int NBW,
                              cudaStream_t st);
// Fused normalise + select writing the row LSE of the scores instead of logG
// (rows of at most 32 * kSelectReg blocks).
cudaError_t launch_normalize_select_compact(const float* s, float* lse, float* tau, int32_t* tau_idx, int32_t* sel,
                                            long long rows, int T, int NB, int H, cudaStream_t st);

// Shape of the query tiles of the tensor-core kernels: P consecutive positions
// of one (b, g) times the G heads of the group, P a multiple of 8 with G*P <= 128.
struct QTileShape {
  int P;         // positions per tile
  int n_ptiles;  // tiles per (b, g)
  int NBW;       // 32-bit words of a per-tile block bitmask
};
QTileShape qtile_shape(int G, int T, int NB);

struct TcProblem {
  int B, Hq, Hkv, T, d, NB, G;
  float sm_scale;
  const void* Q;
  const void* K;
  const void* V;
  const void* O;    // bwd only
  const void* dO;   // bwd only
  const float* logG;      // log gates, or the raw scores s when gate_lse is set
  const float* gate_lse;  // null, or [B*Hkv*T] LSE of each row's historical scores: log g = s - gate_lse
  const float* tau;
  const int32_t* tau_idx;
  const int32_t* sel;  // null, or [B*Hkv*T][K-1] the selection's ascending block lists (-1 padded)
  const float* LSE;  // bwd only
};

// Per-(b, g, block) position lists of the KV-block-outer kernels (sas_lists.cu).
// An entry packs the position (bits 0-17) and the pair's slot in its row (bits
// 18-30): 1 + the block's rank among the row's selected blocks, slot 0 being the
// row's own block.
constexpr int kEntrySlotShift = 18;
constexpr int32_t kEntryPosMask = (1 << kEntrySlotShift) - 1;
struct BlockLists {
  int32_t* cnt;      // [nbg * NB] selecting positions per block
  int32_t* off;      // [nbg * NB] first entry of each block's list
  int32_t* cap;      // [nbg * NB] entries of each list that fit its region
  int32_t* ccnt;     // [nbg * chunks * NB] per-chunk counts, then each chunk's first entry
  int32_t* list;     // [nbg * region] entries
  int32_t* nsel;     // [nbg * T] selected blocks per row (capped at K-1)
  int32_t* total;    // [nbg] entries in use
  long long region;  // entries per (b, g): T * min(K-1, NB)
};
size_t block_lists_bytes(long long nbg, int T, int NB, int K);
BlockLists carve_block_lists(uint8_t* scratch, long long nbg, int T, int NB, int K);
cudaError_t launch_block_lists(const float* logG, const float* gate_lse, const float* tau, const int32_t* tau_idx,
                               const int32_t* sel, const BlockLists& L,
                               long long nbg, int T, int NB, int K, bool want_nsel, int32_t* status,
                               cudaStream_t st);

// bf16 tensor-core forward over the union of each q-tile's blocks; ws holds the
// status word and the tile masks.
cudaError_t launch_fwd_tc(const TcProblem& pb, void* O, float* LSE, int32_t* status, uint32_t* masks,
                          cudaStream_t st);
// bf16 tensor-core forward, KV-block outer over gathered query rows with
// per-(position, block) partials merged per row; `scratch` holds
// fwd_gather_workspace_bytes bytes. fwd_gather_applies: whether the partials of
// one (b, g) fit the slot budget (else the union forward runs).
bool fwd_gather_applies(int B, int Hq, int Hkv, int T, int K);
size_t fwd_gather_workspace_bytes(int B, int Hq, int Hkv, int T, int K);
cudaError_t launch_fwd_gather(const TcProblem& pb, int K, void* O, float* LSE, int32_t* status, uint8_t* scratch,
                              cudaStream_t st);
// bf16 tensor-core backward (KV-block outer, gathered query rows); `scratch`
// holds bwd_gather_workspace_bytes bytes.
size_t bwd_gather_workspace_bytes(int B, int Hq, int Hkv, int T, int K);
cudaError_t launch_bwd_gather(const TcProblem& pb, int K, void* dQ, void* dK, void* dV, float* dLogG, int32_t* status,
                              float* delta, uint8_t* scratch, cudaStream_t st);

// fp32 CUDA-core forward / backward.
cudaError_t launch_fwd_simt(const TcProblem& pb, float* O, float* LSE, cudaStream_t st);
cudaError_t launch_bwd_simt(const TcProblem& pb, float* dQ, float* dK, float* dV, float* dLogG, float* delta,
                            cudaStream_t st);

// Decode (bf16 or fp32 storage).
struct DecodeProblem {
  int B, Hq, Hkv, Lmax, NBmax, d, K, apply_log_gate, dtype;
  float sm_scale;
  const void* q;
  const void* Kc;
  const void* Vc;
  const int32_t* seqlen;
  const float* s;
  void* o;
  int32_t* sel_out;
  const int32_t* page_table = nullptr;   // [B][max_pages]; null: contiguous cache
  int max_pages = 0, num_pages = 0;
};
size_t decode_workspace_bytes(int B, int Hq, int Hkv, int K);
cudaError_t launch_decode(const DecodeProblem& pb, void* ws, cudaStream_t st);
// Decode with the library's own static device scratch instead of a workspace.
size_t decode_static_scratch_limit();
cudaError_t launch_decode_static(const DecodeProblem& pb, cudaStream_t st);
// Synchronises st and reads the status word of the static scratch of the current device.
cudaError_t decode_static_status(cudaStream_t st, int32_t* out);

}  // namespace sas
