// SAS backward, KV-block outer with gathered query rows (sm_100a tensor cores).
//
// SAS paper (arXiv 2609.13141) Appendix E "Backward pass": recompute P from the
// saved LSE, Delta = rowsum(O * dO), dS = P * (dP - Delta); the block log-gate
// gradient is the per-block sum of dS over the block's tokens (summed over the
// G query heads of the group, which share the gate).
//
// The selection is per query row and, for i.i.d. selector scores, rows of one
// q-tile pick nearly disjoint blocks. Instead of running a q-tile over the union
// of its rows' blocks (most of the tile masked), each CTA owns one KV block j of
// one (b, g) and visits exactly the rows that attend it: its own 64 positions
// (causal) and the positions that selected j, gathered P at a time (x G heads
// = up to 128 rows) by cp.async copies of packed chunks. Per tile, on tcgen05:
//   S = Q K_j^T, dP = dO V_j^T              (M = 128 rows, N = 64 keys)
//   dV_j^T += dO^T P, dK_j^T += Q^T dS      (M = 128 features, N = 64 keys, K = rows)
//   dQ_rows = dS K_j                        (M = 128 rows, N = 128 features, K = 64 keys)
// dK_j/dV_j stay in TMEM for the whole CTA; dQ partials leave through fp32
// reductions into a workspace accumulator; dLogG[t, j] is written once, by the
// CTA of block j. Tensor-core work equals the attended work (no union waste).
//
// Delta from the stored (bf16) O is off by the rounding of O. dQ/dK/dV barely
// notice, but dLogG[t, m] = sum_h (A_hm - P_h(B_m) Delta_h), with A_hm the
// block's sum of P dP and P_h(B_m) its probability mass, is a difference of two
// close terms when one selected block holds most of the mass. So each CTA also
// adds its per-head block sum of dS into eps[t, h] (over all attended blocks,
// that is exactly Delta_h - Delta_stored_h, because P sums to one) and stores
// P_h(B_m); a finishing kernel subtracts sum_h P_h(B_m) eps[t, h] from dLogG.
//
// Pre-pass: the per-block position lists of sas_lists.cu, and a pack kernel
// that gathers each position's Q and dO rows of the G heads with LSE and Delta
// into one contiguous chunk.

#include "sas_common.cuh"
#include "sas_kernels.h"
#include "sas_tmap.h"

#include <algorithm>

namespace sas {
namespace gbwd {

constexpr int D = 128;
// Warps 0-3: softmax / dS (one thread per tile row); warp 4: control (K/V
// load; per tile the row positions, then the copies of each row's gate, score
// LSE and chunk tail into a metadata ring that runs up to MST tiles ahead of
// the rows); warp 5: MMA issuer; warps 6-9: dQ flush (TMEM -> shared-memory
// staging -> fp32 reductions of whole row segments); warps 10-15: Q/dO row
// gathers. A Q/dO stage is busy from its gather to the tile's dK/dV MMAs, and
// only two fit in shared memory, so the gather of a tile starts when the tile
// two back has finished: the small scattered metadata loads (with the longest
// latency of the tile's copies) are taken out of that cycle by the metadata
// ring. The gather bandwidth one SM sustains grows with the number of warps
// issuing copies, so most warps load; the softmax works on 32 key columns at a
// time to keep the kernel within 128 registers per thread.
constexpr int THREADS = 512;
constexpr int LOADER_WARP0 = 10, N_LOADER_WARPS = 6;
constexpr int NST = 2;                           // Q/dO gather stages
constexpr int MST = 4;                           // metadata stages
constexpr int MLAG = 2;                          // metadata tiles in flight per control lane beyond the oldest
constexpr uint32_t HALF128 = 128 * 128;          // one d-half of a 128-row tile
constexpr uint32_t TILE = 2 * HALF128;           // 128 rows x 128 features, bf16
constexpr uint32_t KV_HALF = 64 * 128;
constexpr uint32_t OFF_K = 0;
constexpr uint32_t OFF_V = 2 * KV_HALF;
constexpr uint32_t OFF_QD = 4 * KV_HALF;                  // stage s: Q at +2s*TILE, dO at +(2s+1)*TILE
constexpr uint32_t OFF_P = OFF_QD + NST * 2 * TILE;       // P  [128 rows][64 keys] bf16 (16 KiB)
constexpr uint32_t OFF_DS = OFF_P + 128 * 128;            // dS [128 rows][64 keys] bf16 (16 KiB)
// Per metadata stage: the tile's positions [128] int, the gate score of each
// position for block j [128] float and its row's score LSE [128] float (0 unless
// the gates come as raw scores), and the chunk tails (LSE and Delta of the G
// heads) of each position, `tail` bytes apiece (P positions * tail <= 2 KiB for
// every G).
constexpr uint32_t CMETA_STAGE = 2048;
constexpr uint32_t OFF_META = OFF_DS + 128 * 128;
constexpr uint32_t META_STAGE = 3 * 128 * 4;   // positions, gate scores, row score LSEs (compact gates)
constexpr uint32_t OFF_CMETA = OFF_META + MST * META_STAGE;
constexpr uint32_t OFF_QROW = OFF_CMETA + MST * CMETA_STAGE;   // [2][128] global row of each dQ buffer row (-1: none)
constexpr uint32_t OFF_RED = OFF_QROW + 2 * 128 * 4;      // [2][128] fp32 row sums for dLogG
// dQ flush staging: per flush warp one 32-column chunk of its 32 rows (fp32,
// 16-byte pieces XOR-swizzled by row), so that each reduction instruction adds
// whole 128-byte row segments (four rows, four full lines) instead of one
// 16-byte piece of 32 different rows.
constexpr uint32_t OFF_DQS = OFF_RED + 2 * 128 * 4;
constexpr uint32_t DQS_WARP_BYTES = 32 * 128;
constexpr uint32_t OFF_BAR = OFF_DQS + 4 * DQS_WARP_BYTES;
constexpr uint32_t OFF_MISC = OFF_BAR + 256;
constexpr uint32_t SMEM_BYTES = OFF_MISC + 64 + 1024;
static_assert(SMEM_BYTES <= 232448, "shared memory of one CTA");
// TMEM columns
constexpr uint32_t COL_S = 0, COL_DP = 64, COL_DV = 128, COL_DK = 192, COL_DQ0 = 256, TMEM_COLS = 512;

struct Params {
  const float* logG;         // log gates, or raw scores when gate_lse is set
  const float* gate_lse;     // null, or the LSE of each row's historical scores
  const float* tau;
  const int32_t* tau_idx;
  const float* LSE;
  const int32_t* cnt;        // [B*Hkv*NB] selecting rows per block
  const int32_t* off;        // [B*Hkv*NB] start of each block's list
  const int32_t* list;       // entries: position | slot << kEntrySlotShift
  const int32_t* list_cap;   // [B*Hkv*NB] entries of each list that fit its region
  // Packed rows, one chunk of `chunk` bytes per (b, g, position): Q [G][D] bf16,
  // dO [G][D] bf16, then LSE[G] and Delta[G] fp32 (padded to 16 bytes).
  const uint8_t* packed;
  int chunk;
  float* dQacc;              // [B*Hq*T*D] fp32, zeroed before the launch
  __nv_bfloat16* dK;
  __nv_bfloat16* dV;
  float* dLogG;
  float* eps;                // [B*Hkv*T][G] fp32, zeroed: sum over attended blocks of the block dS sums
  float* pmass;              // [list entry][G] probability mass of the entry's block, per head
  int32_t* dl_idx;           // [list entry] t * NB + j of the entry's dLogG element within its (b, g)
  int32_t* status;
  int B, Hq, Hkv, T, NB, G, P;
  int group_major;           // CTA order: 1 group-major, 0 block-major
  float scale_log2;
  float sm_scale;
  uint64_t wait_ns;          // limit of one bounded wait
};

struct Bars {
  uint64_t kv_full, pos_ready[MST], meta_full[MST], meta_empty[MST], qd_full[NST], qd_empty[NST], s_full, sp_free,
      p_full, pd_free, dq_done[2], dq_free[2], qrow_full[2], fin;
};
static_assert(sizeof(Bars) <= 256, "barrier area");

// Position of list entry `idx` of block j: the block's own positions first, then the selecting rows.
__device__ __forceinline__ int tile_position(const int32_t* lst, int own_n, int total, int j, int idx) {
  if (idx >= total) return -1;
  return idx < own_n ? j * kBlock + idx : (lst[idx - own_n] & kEntryPosMask);
}

// One flush warp's 32 rows of a dQ partial (TMEM lanes of its quarter) into the
// fp32 accumulator, 32 columns at a time through the warp's staging area.
// qrows: this warp's 32 entries of the buffer's row map (-1: no row).
__device__ __forceinline__ void flush_dq(const Params& p, uint32_t taddr, const int* qrows, uint8_t* stage) {
  const int lane = threadIdx.x & 31;
#pragma unroll 1
  for (int ch = 0; ch < D / 32; ++ch) {
    uint32_t v[32];
    tmem_ld32(taddr + 32 * ch, v);
    tmem_wait_ld();
#pragma unroll
    for (int k = 0; k < 8; ++k)
      *reinterpret_cast<uint4*>(stage + lane * 128 + ((k ^ (lane & 7)) << 4)) =
          make_uint4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
    __syncwarp();
#pragma unroll
    for (int m = 0; m < 8; ++m) {   // rows 4m .. 4m+3, eight lanes per row
      const int rr = 4 * m + (lane >> 3), k = lane & 7;
      const int qrow = qrows[rr];
      if (qrow >= 0) {
        const float4 x = *reinterpret_cast<const float4*>(stage + rr * 128 + ((k ^ (rr & 7)) << 4));
        red_add_v4(p.dQacc + (long long)qrow * D + 32 * ch + 4 * k, x.x, x.y, x.z, x.w);
      }
    }
    __syncwarp();
  }
}

__global__ void __launch_bounds__(THREADS, 1)
    sas_bwd_gather_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                          const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars* bars = reinterpret_cast<Bars*>(smem + OFF_BAR);
  int* qrow_s = reinterpret_cast<int*>(smem + OFF_QROW);
  float* red = reinterpret_cast<float*>(smem + OFF_RED);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_MISC);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // CTA order. Block j is attended by its own positions and by the later
  // positions that select it, so small j carry the longest row lists. Group-major
  // order (all blocks of (b, g) 0, then of (b, g) 1, ...) keeps the rows that the
  // running CTAs gather and reduce into within about one group, which fits L2
  // far better than all groups' (DRAM traffic of the 32K-token layer: 14 GB
  // instead of 61 GB), but the last group's long lists start late. That tail
  // matters when a group is less than two waves of CTAs; those problems run
  // block-major (every group's block 0, then block 1, ...), which starts all
  // long lists first.
  const int n_bg = p.B * p.Hkv;
  const int bg = p.group_major ? (int)(blockIdx.x / p.NB) : (int)(blockIdx.x % n_bg);
  const int j = p.group_major ? (int)(blockIdx.x % p.NB) : (int)(blockIdx.x / n_bg);
  const uint64_t wait_ns = p.wait_ns;
  const int b = bg / p.Hkv, g = bg % p.Hkv;
  const int PP = p.P, G = p.G;
  const int rows_used = G * PP;
  const int own_n = min(kBlock, p.T - j * kBlock);
  const int sel_n = min(p.cnt[(long long)bg * p.NB + j], p.list_cap[(long long)bg * p.NB + j]);
  const int total = own_n + sel_n;
  const int n_tiles = (total + PP - 1) / PP;
  const long long off_j = p.off[(long long)bg * p.NB + j];
  const int32_t* lst = p.list + off_j;
  int32_t* status = p.status;

  if (warp == 5) tmem_alloc(tmem_slot, TMEM_COLS);
  if (tid == 0) {
    mbar_init(&bars->kv_full, 1);
    for (int i = 0; i < MST; ++i) {
      mbar_init(&bars->pos_ready[i], 1);
      mbar_init(&bars->meta_full[i], 1);
      mbar_init(&bars->meta_empty[i], 4);   // softmax warps
    }
    for (int i = 0; i < NST; ++i) {
      mbar_init(&bars->qd_full[i], N_LOADER_WARPS);
      mbar_init(&bars->qd_empty[i], 1);
    }
    mbar_init(&bars->s_full, 1);
    mbar_init(&bars->sp_free, 4);
    mbar_init(&bars->p_full, 4);
    mbar_init(&bars->pd_free, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->dq_done[i], 1);
      mbar_init(&bars->dq_free[i], 4);
      mbar_init(&bars->qrow_full[i], 4);
    }
    mbar_init(&bars->fin, 1);
    fence_barrier_init();
  }
  if (rows_used < 128) {   // rows never gathered stay zero
    const int per = (128 - rows_used) * 8;
    for (int i = tid; i < per * 2 * 2 * NST; i += THREADS) {
      const int tile = i / (2 * per), half = (i / per) & 1, rem = i % per;
      *reinterpret_cast<uint4*>(smem + OFF_QD + tile * TILE + half * HALF128 + (rows_used + rem / 8) * 128 +
                                (rem % 8) * 16) = make_uint4(0, 0, 0, 0);
    }
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t s_base = smem_u32(smem);

  if (warp == 4) {
    // ------------------------------------------------------------------ control: positions + metadata
    if (lane == 0) {
      mbar_expect_tx(&bars->kv_full, 4 * KV_HALF);
      tma_load_3d(smem + OFF_K, &tmK, &bars->kv_full, 0, j * kBlock, bg);
      tma_load_3d(smem + OFF_K + KV_HALF, &tmK, &bars->kv_full, 64, j * kBlock, bg);
      tma_load_3d(smem + OFF_V, &tmV, &bars->kv_full, 0, j * kBlock, bg);
      tma_load_3d(smem + OFF_V + KV_HALF, &tmV, &bars->kv_full, 64, j * kBlock, bg);
    }
    // Positions of tile i (own positions first, then the list; -1 past the end).
    // The next tile's are loaded while the current one is published.
    auto load_pos = [&](int i, int (&tl)[4]) {
#pragma unroll
      for (int u = 0; u < 4; ++u)
        tl[u] = (lane + 32 * u < PP) ? tile_position(lst, own_n, total, j, i * PP + lane + 32 * u) : -1;
    };
    const int tail_bytes = p.chunk - 512 * G;   // LSE and Delta of the G heads, padded to 16 bytes
    const uint8_t* base = p.packed + (long long)bg * p.T * p.chunk;
    int cur[4], nxt[4] = {-1, -1, -1, -1};
    load_pos(0, cur);
    int issued = 0;
    for (int i = 0; i < n_tiles; ++i) {
      const int ms = i % MST;
      if (i + 1 < n_tiles) load_pos(i + 1, nxt);
      bool ok = true;
      if (i >= MST) ok = mbar_wait(&bars->meta_empty[ms], ((i / MST) - 1) & 1, status, wait_ns);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      int* pos = reinterpret_cast<int*>(smem + OFF_META + ms * META_STAGE);
      float* gate = reinterpret_cast<float*>(pos + 128);
      float* glse = gate + 128;
      const uint32_t cm = s_base + OFF_CMETA + ms * CMETA_STAGE;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int pp = lane + 32 * u;
        if (pp >= PP) continue;
        const int t = cur[u];
        pos[pp] = t;
        // The gate of block j for each selecting position (0 for own positions and
        // empty slots), with its row's score LSE when the gates come as raw scores.
        if (t >= 0 && t / kBlock != j) {
          cp_async4(smem_u32(gate + pp), p.logG + ((long long)bg * p.T + t) * p.NB + j);
          if (p.gate_lse)
            cp_async4(smem_u32(glse + pp), p.gate_lse + (long long)bg * p.T + t);
          else
            glse[pp] = 0.f;
        } else {
          gate[pp] = 0.f;
          glse[pp] = 0.f;
        }
        if (t >= 0)
          for (int k = 0; k < tail_bytes; k += 16)
            cp_async16(cm + pp * tail_bytes + k, base + (long long)t * p.chunk + 512 * G + k);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->pos_ready[ms]);
      cp_async_commit();
      ++issued;
      // Tile i-MLAG's metadata is published once it has landed, with the copies of
      // tiles i-MLAG+1 .. i still in flight.
      if (i >= MLAG) {
        cp_async_wait_group<MLAG>();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->meta_full[(i - MLAG) % MST]);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) cur[u] = nxt[u];
    }
    cp_async_wait_all();   // after a failed wait too: no copy may outlive the CTA
    __syncwarp();
    if (lane == 0)
      for (int k = max(0, issued - MLAG); k < issued; ++k) mbar_arrive(&bars->meta_full[k % MST]);
    if (lane == 0) mbar_wait_drain(&bars->kv_full, 0);
  } else if (warp >= LOADER_WARP0) {
    // ------------------------------------------------------------------ loaders: Q / dO row gathers
    const int lt = tid - LOADER_WARP0 * 32;
    constexpr int NL = N_LOADER_WARPS * 32;
    // Pieces of 16 bytes of the Q/dO rows of each position's chunk: 32*G of them
    // (ordered tensor, head, piece), piece lt + k * NL of the tile for this
    // thread, so consecutive lanes copy consecutive bytes. The map from a piece to
    // its tile position, shared-memory offset and offset in the chunk is the same
    // for every tile: it is taken once, and a tile then only reads its positions.
    constexpr int MAXP = (128 * 32 + NL - 1) / NL;   // G * P <= 128 rows of 16 pieces, Q and dO
    const int rows_pieces = 32 * G;
    const int n_pieces = PP * rows_pieces;
    int pk_pp[MAXP];
    uint32_t pk_dst[MAXP], pk_src[MAXP];
#pragma unroll
    for (int k = 0; k < MAXP; ++k) {
      const int piece = lt + k * NL;
      const int pp = piece < n_pieces ? piece / rows_pieces : 0;
      const int rem = piece < n_pieces ? piece - pp * rows_pieces : 0;
      const int tensor = rem >= 16 * G;
      const int rem2 = rem - tensor * 16 * G;
      const int hh = rem2 >> 4, c16 = rem2 & 15;
      pk_pp[k] = piece < n_pieces ? pp : -1;
      pk_dst[k] = (uint32_t)tensor * TILE + (uint32_t)(c16 >> 3) * HALF128 +
                  sw128_offset((uint32_t)(hh * PP + pp), (uint32_t)(c16 & 7));
      pk_src[k] = (uint32_t)rem * 16;
    }
    const uint8_t* base = p.packed + (long long)bg * p.T * p.chunk;
    for (int i = 0; i < n_tiles; ++i) {
      const int st = i % NST, ms = i % MST;
      bool ok = true;
      if (i >= NST) ok = mbar_wait(&bars->qd_empty[st], ((i / NST) - 1) & 1, status, wait_ns);
      if (ok) ok = mbar_wait(&bars->pos_ready[ms], (i / MST) & 1, status, wait_ns);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      const int* pos = reinterpret_cast<const int*>(smem + OFF_META + ms * META_STAGE);
      const int first = pos[0];
      const uint32_t qd = s_base + OFF_QD + st * 2 * TILE;
#pragma unroll
      for (int k = 0; k < MAXP; ++k) {
        if (pk_pp[k] < 0) continue;
        const int t0 = pos[pk_pp[k]];
        cp_async16(qd + pk_dst[k], base + (long long)(t0 >= 0 ? t0 : first) * p.chunk + pk_src[k]);
      }
      cp_async_commit_wait_all();
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->qd_full[st]);
    }
    cp_async_wait_all();   // after a failed wait too: no copy may outlive the CTA
  } else if (warp == 5) {
    // ------------------------------------------------------------------ MMA issuer
    // A polling state machine: S/dP of the next tile and dV/dK/dQ of the oldest
    // tile are issued as soon as their inputs are ready, in whichever order.
    if (lane == 0) {
      const uint32_t idesc_s = make_idesc_bf16(128, 64, 0, 0);    // rows x keys, K = features
      const uint32_t idesc_t = make_idesc_bf16(128, 64, 1, 1);    // features x keys, K = rows
      const uint32_t idesc_q = make_idesc_bf16(128, D, 0, 1);     // rows x features, K = keys
      // Shared-memory descriptors: the address field is the byte address / 16, so
      // an operand at base + off (off a multiple of 16, inside the 256 KiB the
      // field spans) has descriptor desc(base) + off / 16. The bases are taken
      // once; each MMA adds a constant.
      const uint64_t d_k = make_sdesc(s_base + OFF_K, 16, 1024);             // K_j, K-major (S, dQ's B below)
      const uint64_t d_v = make_sdesc(s_base + OFF_V, 16, 1024);             // V_j, K-major
      const uint64_t d_qd = make_sdesc(s_base + OFF_QD, 16, 1024);           // stage 0 Q; dO at + TILE
      const uint64_t d_qd_t = make_sdesc(s_base + OFF_QD, HALF128, 1024);    // the same, MN-major
      const uint64_t d_p_t = make_sdesc(s_base + OFF_P, HALF128, 1024);
      const uint64_t d_ds_t = make_sdesc(s_base + OFF_DS, HALF128, 1024);
      const uint64_t d_ds = make_sdesc(s_base + OFF_DS, 16, 1024);
      const uint64_t d_k_q = make_sdesc(s_base + OFF_K, KV_HALF, 1024);
      bool ok = mbar_wait(&bars->kv_full, 0, status, wait_ns);
      int ns = 0, nb = 0;
      uint64_t t_last = global_ns();
      uint32_t spins = 0;
      while (ok && nb < n_tiles) {
        bool prog = false;
        if (ns < n_tiles) {
          const int st = ns % NST;
          if (mbar_test_wait(&bars->qd_full[st], (ns / NST) & 1) &&
              (ns == 0 || mbar_test_wait(&bars->sp_free, (ns - 1) & 1))) {
            tc_fence_after();
            const uint64_t qs = (uint64_t)(st * 2 * TILE) >> 4;   // this stage's offset in descriptor units
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
              const uint32_t half = ks >> 2, koff = (ks & 3) * 32;
              umma_ss(tmem + COL_S, d_qd + qs + ((half * HALF128 + koff) >> 4), d_k + ((half * KV_HALF + koff) >> 4),
                      idesc_s, ks > 0 ? 1u : 0u);
            }
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
              const uint32_t half = ks >> 2, koff = (ks & 3) * 32;
              umma_ss(tmem + COL_DP, d_qd + qs + ((TILE + half * HALF128 + koff) >> 4),
                      d_v + ((half * KV_HALF + koff) >> 4), idesc_s, ks > 0 ? 1u : 0u);
            }
            umma_commit(&bars->s_full);
            ++ns;
            prog = true;
          }
        }
        if (nb < ns && mbar_test_wait(&bars->p_full, nb & 1) &&
            (nb < 2 || mbar_test_wait(&bars->dq_free[nb & 1], ((nb - 2) >> 1) & 1))) {
          tc_fence_after();
          const int st = nb % NST, qb_ = nb & 1;
          const uint64_t qs = (uint64_t)(st * 2 * TILE) >> 4;
#pragma unroll
          for (int ks = 0; ks < 8; ++ks) {   // K = 128 rows, 16 per MMA
            umma_ss(tmem + COL_DV, d_qd_t + qs + ((TILE + ks * 2048) >> 4), d_p_t + ((ks * 2048) >> 4), idesc_t,
                    (nb > 0 || ks > 0) ? 1u : 0u);
          }
#pragma unroll
          for (int ks = 0; ks < 8; ++ks) {
            umma_ss(tmem + COL_DK, d_qd_t + qs + ((ks * 2048) >> 4), d_ds_t + ((ks * 2048) >> 4), idesc_t,
                    (nb > 0 || ks > 0) ? 1u : 0u);
          }
          umma_commit(&bars->qd_empty[st]);
#pragma unroll
          for (int ks = 0; ks < 4; ++ks) {   // dQ partial = dS K_j, K = 64 keys
            umma_ss(tmem + COL_DQ0 + 128 * qb_, d_ds + ((ks * 32) >> 4), d_k_q + ((ks * 2048) >> 4), idesc_q,
                    ks > 0 ? 1u : 0u);
          }
          umma_commit(&bars->dq_done[qb_]);
          umma_commit(&bars->pd_free);
          ++nb;
          prog = true;
        }
        if (prog) {
          t_last = global_ns();
          spins = 0;
        } else if ((++spins & 255u) == 0u) {
          if (*reinterpret_cast<volatile int32_t*>(status) != 0) break;
          if (global_ns() - t_last > wait_ns) {
            set_status(status, SAS_DEV_ERR_TIMEOUT);
            break;
          }
        }
      }
      umma_commit(&bars->fin);
      mbar_wait_drain(&bars->fin, 0);
    }
  } else if (warp >= 6) {
    // ------------------------------------------------------------------ dQ flush (warps 6-9)
    const int quarter = warp & 3;                    // TMEM lanes this warp may access
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    for (int i = 0; i < n_tiles; ++i) {
      const int qb = i & 1;
      if (!warp_wait(&bars->qrow_full[qb], (i >> 1) & 1, status, wait_ns)) break;
      if (!warp_wait(&bars->dq_done[qb], (i >> 1) & 1, status, wait_ns)) break;
      tc_fence_after();
      flush_dq(p, tmem + lane_base + COL_DQ0 + 128 * qb, qrow_s + qb * 128 + quarter * 32,
               smem + OFF_DQS + quarter * DQS_WARP_BYTES);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->dq_free[qb]);
    }
  } else {
    // ------------------------------------------------------------------ softmax / dS (warps 0-3)
    const int r = tid;
    const int hh = r / PP;
    const int h = g * G + (hh < G ? hh : 0);
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    bool ok = true;
    for (int i = 0; i < n_tiles; ++i) {
      const int st = i % NST, ms = i % MST, qb = i & 1;
      bool step_ok = warp_wait(&bars->meta_full[ms], (i / MST) & 1, status, wait_ns);
      if (step_ok) step_ok = warp_wait(&bars->qd_full[st], (i / NST) & 1, status, wait_ns);
      int t = -1;
      float lse2 = 0.f, dlt = 0.f, bias2 = 0.f;
      if (step_ok && r < rows_used) {
        const int pp = r % PP;
        t = reinterpret_cast<const int*>(smem + OFF_META + ms * META_STAGE)[pp];
        if (t >= 0) {
          const float* tail =
              reinterpret_cast<const float*>(smem + OFF_CMETA + ms * CMETA_STAGE + pp * (p.chunk - 512 * G));
          lse2 = tail[hh] * kLog2e;
          dlt = tail[G + hh];
          // log g = s - LSE(s) in fp32 (bit-identical to the normalised gate), then log2 units
          const float* gm = reinterpret_cast<const float*>(smem + OFF_META + ms * META_STAGE + 128 * 4);
          bias2 = (gm[pp] - gm[128 + pp]) * kLog2e;
        }
      }
      // The metadata stage is read (and the loaders, done with tile i, read its
      // positions before): the control warp may refill it.
      __syncwarp();
      if (step_ok && lane == 0) mbar_arrive(&bars->meta_empty[ms]);
      const bool valid = step_ok && t >= 0;
      const bool own = valid && (t / kBlock == j);
      const int lim = own ? t - j * kBlock : 63;
      if (step_ok) step_ok = warp_wait(&bars->s_full, i & 1, status, wait_ns);
      // Two passes of 32 key columns: S, dP -> P, dS (bf16) into shared memory.
      if (step_ok) tc_fence_after();
      if (step_ok && i >= 1) {
        // P / dS shared tiles are free once tile i-1's MMAs completed.
        step_ok = warp_wait(&bars->pd_free, (i - 1) & 1, status, wait_ns);
      }
      float rs = 0.f, pm = 0.f;
      if (step_ok) {
#pragma unroll 1
        for (int hc = 0; hc < 2; ++hc) {
          uint32_t sr[32], dr[32];
          tmem_ld32(tmem + lane_base + COL_S + 32 * hc, sr);
          tmem_ld32(tmem + lane_base + COL_DP + 32 * hc, dr);
          tmem_wait_ld();
          if (hc == 1) {   // S / dP of this tile fully read: the next tile's S may overwrite them
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->sp_free);
          }
#pragma unroll
          for (int ch = 0; ch < 4; ++ch) {
            uint32_t pw[4], sw[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              float pv[2], dv[2];
#pragma unroll
              for (int e = 0; e < 2; ++e) {
                const int kk = ch * 8 + 2 * k + e;       // column within this half
                const float sv = __uint_as_float(sr[kk]);
                const float dp = __uint_as_float(dr[kk]);
                pv[e] = (valid && 32 * hc + kk <= lim) ? ex2(fmaf(sv, p.scale_log2, bias2) - lse2) : 0.f;
                dv[e] = pv[e] * (dp - dlt);
                rs += dv[e];
                pm += pv[e];
              }
              pw[k] = pack_bf16(pv[0], pv[1]);
              sw[k] = pack_bf16(dv[0], dv[1]);
            }
            const uint32_t o = sw128_offset((uint32_t)r, (uint32_t)(4 * hc + ch));
            *reinterpret_cast<uint4*>(smem + OFF_P + o) = make_uint4(pw[0], pw[1], pw[2], pw[3]);
            *reinterpret_cast<uint4*>(smem + OFF_DS + o) = make_uint4(sw[0], sw[1], sw[2], sw[3]);
          }
        }
        fence_proxy_async_smem();
      }
      // The dQ row map of buffer qb is reusable once tile i-2 was flushed.
      if (step_ok && i >= 2) step_ok = warp_wait(&bars->dq_free[qb], ((i - 2) >> 1) & 1, status, wait_ns);
      if (step_ok) {
        qrow_s[qb * 128 + r] = valid ? (int)(((long long)b * p.Hq + h) * p.T + t) : -1;
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&bars->qrow_full[qb]);
          mbar_arrive(&bars->p_full);
        }
      }
      // Delta correction terms: this block's dS sum into eps[t, hh]; for a selected
      // block also its probability mass, at the row's list entry.
      if (step_ok && valid) {
        atomicAdd(p.eps + ((long long)bg * p.T + t) * G + hh, rs);
        if (!own) {
          const long long e = off_j + i * PP + (r % PP) - own_n;
          p.pmass[e * G + hh] = pm;
          if (hh == 0) p.dl_idx[e] = t * p.NB + j;
        }
      }
      // dLogG[t, j] for positions that selected j: sum over the G heads (rows hh*PP + pp).
      red[qb * 128 + r] = (valid && !own) ? rs : 0.f;
      ok = named_bar_and(1, 128, step_ok);
      if (!ok) break;
      if (r < PP && valid && !own) {
        float acc = 0.f;
        for (int q = 0; q < G; ++q) acc += red[qb * 128 + q * PP + r];
        p.dLogG[((long long)bg * p.T + t) * p.NB + j] = acc;
      }
    }
    if (ok && n_tiles > 0) ok = warp_wait(&bars->pd_free, (n_tiles - 1) & 1, status, wait_ns);
    if (ok) {
      tc_fence_after();
      const int dd = r;   // TMEM lane = feature
      const long long key0 = (long long)bg * p.T + (long long)j * kBlock;
#pragma unroll 1
      for (int which = 0; which < 2; ++which) {
        const uint32_t col = which == 0 ? COL_DV : COL_DK;
        __nv_bfloat16* dst = which == 0 ? p.dV : p.dK;
        const float scl = which == 0 ? 1.f : p.sm_scale;
#pragma unroll 1
        for (int ch = 0; ch < 2; ++ch) {
          uint32_t v[32];
          tmem_ld32(tmem + lane_base + col + 32 * ch, v);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 32; ++k) {
            const int key = 32 * ch + k;
            if (key < own_n)
              dst[(key0 + key) * D + dd] = __float2bfloat16_rn(n_tiles > 0 ? __uint_as_float(v[k]) * scl : 0.f);
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

// ---------------------------------------------------------------------------- pre-pass
// Packs the rows of each (b, g, position) into one chunk: Q [G][D], dO [G][D]
// (bf16), LSE [G] and Delta [G] = rowsum(O * dO) (fp32). One warp per (b, g, t, head).
__global__ void __launch_bounds__(256) pack_kernel(const __nv_bfloat16* __restrict__ Q,
                                                   const __nv_bfloat16* __restrict__ dO,
                                                   const __nv_bfloat16* __restrict__ O, const float* __restrict__ LSE,
                                                   uint8_t* __restrict__ packed, long long n_rows, int T, int G, int Hq,
                                                   int Hkv, int chunk) {
  const long long w = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);   // (bg, t, hh)
  const int lane = threadIdx.x & 31;
  if (w >= n_rows) return;
  const int hh = (int)(w % G);
  const long long bt = w / G;
  const int t = (int)(bt % T);
  const long long bg = bt / T;
  const long long b = bg / Hkv, g = bg % Hkv;
  const long long row = (b * Hq + g * G + hh) * T + t;
  const uint2 q = *reinterpret_cast<const uint2*>(Q + row * D + lane * 4);
  const uint2 d = *reinterpret_cast<const uint2*>(dO + row * D + lane * 4);
  const uint2 o = *reinterpret_cast<const uint2*>(O + row * D + lane * 4);
  uint8_t* c = packed + bt * chunk;
  *reinterpret_cast<uint2*>(c + hh * D * 2 + lane * 8) = q;
  *reinterpret_cast<uint2*>(c + (G + hh) * D * 2 + lane * 8) = d;
  const __nv_bfloat162* d2 = reinterpret_cast<const __nv_bfloat162*>(&d);
  const __nv_bfloat162* o2 = reinterpret_cast<const __nv_bfloat162*>(&o);
  float acc = 0.f;
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const float2 x = __bfloat1622float2(o2[k]);
    const float2 y = __bfloat1622float2(d2[k]);
    acc = fmaf(x.x, y.x, acc);
    acc = fmaf(x.y, y.y, acc);
  }
#pragma unroll
  for (int off = 16; off; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (lane == 0) {
    float* tail = reinterpret_cast<float*>(c + 2 * G * D * 2);
    tail[hh] = LSE[row];
    tail[G + hh] = acc;
  }
}

__global__ void __launch_bounds__(256) dq_convert_kernel(const float* __restrict__ acc, __nv_bfloat16* __restrict__ dq,
                                                         long long n4, float scale) {
  const long long i = (long long)blockIdx.x * 256 + threadIdx.x;
  if (i >= n4) return;
  const float4 v = reinterpret_cast<const float4*>(acc)[i];
  uint2 o;
  o.x = pack_bf16(v.x * scale, v.y * scale);
  o.y = pack_bf16(v.z * scale, v.w * scale);
  reinterpret_cast<uint2*>(dq)[i] = o;
}

// dLogG[t, j] -= sum_h P_h(B_j) eps[t, h] for every (position, selected block)
// pair: one thread per list entry.
__global__ void __launch_bounds__(256) dlogg_fix_kernel(const int32_t* __restrict__ total,
                                                        const int32_t* __restrict__ dl_idx,
                                                        const float* __restrict__ pmass,
                                                        const float* __restrict__ eps, float* __restrict__ dLogG,
                                                        long long n_entries, long long region, int T, int NB, int G) {
  const long long e = (long long)blockIdx.x * 256 + threadIdx.x;
  if (e >= n_entries) return;
  const long long bg = e / region;
  if (e - bg * region >= total[bg]) return;
  const int idx = dl_idx[e];
  const int t = idx / NB;
  const float* pm = pmass + e * G;
  const float* ep = eps + (bg * T + t) * G;
  float corr = 0.f;
  for (int h = 0; h < G; ++h) corr = fmaf(pm[h], ep[h], corr);
  dLogG[bg * T * NB + idx] -= corr;
}

}  // namespace gbwd

// Bytes of one packed position: Q and dO rows of the G heads, then LSE and Delta padded to 16 bytes.
static size_t packed_chunk_bytes(int G) { return (size_t)4 * G * 128 + ((size_t)8 * G + 15) / 16 * 16; }

size_t bwd_gather_workspace_bytes(int B, int Hq, int Hkv, int T, int K) {
  const int NB = T / kBlock;
  const long long nbg = (long long)B * Hkv;
  const long long region = (long long)T * max(1, min(K - 1, NB));
  auto a256 = [](size_t x) { return (x + 255) / 256 * 256; };
  size_t n = 0;
  n += a256((size_t)B * Hq * T * 128 * sizeof(float));     // dQ accumulator
  n += block_lists_bytes(nbg, T, NB, K);                   // per-block position lists
  n += a256((size_t)B * Hkv * T * packed_chunk_bytes(Hq / Hkv));   // packed rows
  n += a256((size_t)B * Hq * T * sizeof(float));           // eps [B*Hkv*T][G]
  n += a256((size_t)nbg * region * (Hq / Hkv) * sizeof(float));    // pmass, one per list entry and head
  n += a256((size_t)nbg * region * sizeof(int32_t));       // dLogG element of each list entry
  return n;
}

cudaError_t launch_bwd_gather(const TcProblem& pb, int K, void* dQ, void* dK, void* dV, float* dLogG, int32_t* status,
                              float* delta, uint8_t* scratch, cudaStream_t st) {
  using namespace gbwd;
  (void)delta;
  const int NB = pb.NB;
  const long long nbg = (long long)pb.B * pb.Hkv;
  const long long rows = nbg * pb.T;
  const long long qrows = (long long)pb.B * pb.Hq * pb.T;
  auto a256 = [](size_t x) { return (x + 255) / 256 * 256; };
  float* dQacc = reinterpret_cast<float*>(scratch);
  size_t o = a256((size_t)qrows * D * sizeof(float));
  const BlockLists L = carve_block_lists(scratch + o, nbg, pb.T, NB, K);
  o += block_lists_bytes(nbg, pb.T, NB, K);
  const long long region = L.region;
  uint8_t* packed = scratch + o;
  const int chunk = (int)packed_chunk_bytes(pb.G);
  o += a256((size_t)rows * chunk);
  float* eps = reinterpret_cast<float*>(scratch + o);
  o += a256((size_t)qrows * sizeof(float));
  float* pmass = reinterpret_cast<float*>(scratch + o);
  o += a256((size_t)nbg * region * pb.G * sizeof(float));
  int32_t* dl_idx = reinterpret_cast<int32_t*>(scratch + o);

  cudaError_t e;
  if ((e = cudaMemsetAsync(dLogG, 0, (size_t)rows * NB * sizeof(float), st)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(dQacc, 0, (size_t)qrows * D * sizeof(float), st)) != cudaSuccess) return e;
  if ((e = cudaMemsetAsync(eps, 0, (size_t)qrows * sizeof(float), st)) != cudaSuccess) return e;
  if ((e = launch_block_lists(pb.logG, pb.gate_lse, pb.tau, pb.tau_idx, pb.sel, L, nbg, pb.T, NB, K, false, status,
                              st)) != cudaSuccess)
    return e;
  pack_kernel<<<(unsigned)((qrows + 7) / 8), 256, 0, st>>>(
      reinterpret_cast<const __nv_bfloat16*>(pb.Q), reinterpret_cast<const __nv_bfloat16*>(pb.dO),
      reinterpret_cast<const __nv_bfloat16*>(pb.O), pb.LSE, packed, qrows, pb.T, pb.G, pb.Hq, pb.Hkv, chunk);
  count_launch();
  if ((e = cudaGetLastError()) != cudaSuccess) return e;

  const QTileShape qs = qtile_shape(pb.G, pb.T, NB);
  CUtensorMap tk, tv;
  if (!make_tmap_bf16_3d(&tk, pb.K, pb.d, pb.T, (uint64_t)nbg, 64) ||
      !make_tmap_bf16_3d(&tv, pb.V, pb.d, pb.T, (uint64_t)nbg, 64))
    return cudaErrorInvalidValue;
  Params prm;
  prm.logG = pb.logG;
  prm.gate_lse = pb.gate_lse;
  prm.tau = pb.tau;
  prm.tau_idx = pb.tau_idx;
  prm.LSE = pb.LSE;
  prm.cnt = L.cnt;
  prm.off = L.off;
  prm.list = L.list;
  prm.list_cap = L.cap;
  prm.dQacc = dQacc;
  prm.packed = packed;
  prm.chunk = chunk;
  prm.dK = reinterpret_cast<__nv_bfloat16*>(dK);
  prm.dV = reinterpret_cast<__nv_bfloat16*>(dV);
  prm.dLogG = dLogG;
  prm.eps = eps;
  prm.pmass = pmass;
  prm.dl_idx = dl_idx;
  prm.status = status;
  prm.B = pb.B;
  prm.Hq = pb.Hq;
  prm.Hkv = pb.Hkv;
  prm.T = pb.T;
  prm.NB = NB;
  prm.G = pb.G;
  prm.P = qs.P;
  int dev = 0, n_sm = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
  prm.group_major = NB >= 2 * n_sm ? 1 : 0;
  prm.scale_log2 = pb.sm_scale * kLog2e;
  prm.sm_scale = pb.sm_scale;
  prm.wait_ns = wait_limit_ns();
  if ((e = cudaFuncSetAttribute(sas_bwd_gather_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES)) !=
      cudaSuccess)
    return e;
  sas_bwd_gather_kernel<<<(unsigned)(nbg * NB), THREADS, SMEM_BYTES, st>>>(tk, tv, prm);
  count_launch();
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  dlogg_fix_kernel<<<(unsigned)((nbg * region + 255) / 256), 256, 0, st>>>(L.total, dl_idx, pmass, eps, dLogG,
                                                                          nbg * region, region, pb.T, NB, pb.G);
  count_launch();
  const long long n4 = qrows * D / 4;
  dq_convert_kernel<<<(unsigned)((n4 + 255) / 256), 256, 0, st>>>(dQacc, reinterpret_cast<__nv_bfloat16*>(dQ), n4,
                                                                  pb.sm_scale);
  count_launch();
  return cudaGetLastError();
}

}  // namespace sas
