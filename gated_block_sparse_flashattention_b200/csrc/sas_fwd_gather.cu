// SAS forward, KV-block outer with gathered query rows (sm_100a tensor cores).
//
// SAS paper (arXiv 2609.13141) §4.3 eq. 9 and Appendix E "Forward pass": row t
// attends its own block (causal, unbiased) and the selected historical blocks,
// each with the row's log gate added to its logits.
//
// With i.i.d. selector scores the rows of a q-tile select nearly disjoint
// blocks, so a q-tile scanning the union of its rows' blocks executes several
// times the attended work (about 8x at 32K tokens, 16x at 64K). Here the CTA of
// block j of (b, g) instead visits exactly the rows that attend j: its own 64
// positions and the positions that selected it (lists from sas_lists.cu),
// gathered P at a time (x G heads = up to 128 rows). Per tile, on tcgen05:
//   S = Q K_j^T        (M = 128 rows, N = 64 keys, K = 128 features)
//   O_j = P V_j        (A = P from TMEM, M = 128 rows, N = 128 features, K = 64)
// with the softmax of the tile's rows taken over block j alone. Every
// (position, block) pair leaves a partial: the normalised O_j (bf16) and its
// log-sum-exp, in the slot the lists assign (slot 0: the own block, then the
// selected blocks in ascending order). A merge kernel combines a row's slots:
//   LSE = log sum_s exp(lse_s),  O = sum_s exp(lse_s - LSE) O_s,
// which is the softmax over the union of the row's blocks. Tensor-core work is
// the attended work; the cost moves to the partials (about 1 KB per pair for
// G = 4), written once and read once.
//
// Warp roles (512 threads, one CTA per SM):
//   warps 0-3   softmax: one thread per tile row (TMEM lane), P -> TMEM as bf16;
//   warps 4-7   epilogue: O_j rows TMEM -> bf16 -> shared-memory staging ->
//               whole-row stores of the partials to global memory;
//   warp 8      control: K_j/V_j by TMA, then per tile the positions and slots
//               (the next tile's list entries loaded while the current one is published);
//   warp 9      MMA issuer (one thread);
//   warps 10-15 loaders: cp.async gathers of the tile's Q rows and of each row's
//               gate (4-stage ring, three tiles in flight per thread).
// TMEM: two S/P buffers (64 columns each) and two O buffers (128 each), so the
// epilogue of tile i overlaps the softmax of tile i+1 and the MMAs of tile i+2.
#include <algorithm>

#include "sas_common.cuh"
#include "sas_kernels.h"
#include "sas_tmap.h"

namespace sas {
namespace gfwd {

constexpr int D = 128;
constexpr int THREADS = 512;
constexpr int EPI_WARP0 = 4, CTRL_WARP = 8, MMA_WARP = 9, LOADER_WARP0 = 10, N_LOADER_WARPS = 6;
constexpr int NST = 4;                           // Q gather stages
constexpr int LAG = NST - 1;                     // tiles a loader thread has in flight beyond the oldest
constexpr uint32_t HALF128 = 128 * 128;          // one d-half of a 128-row tile (16 KiB)
constexpr uint32_t QTILE = 2 * HALF128;          // 128 rows x 128 features, bf16
constexpr uint32_t KV_HALF = 64 * 128;           // 64 keys x 64 features, bf16
constexpr uint32_t OFF_K = 0;
constexpr uint32_t OFF_V = 2 * KV_HALF;
constexpr uint32_t OFF_Q = 4 * KV_HALF;          // stage s at OFF_Q + s * QTILE
// Per stage: position [128] int, gate score of block j [128] float, slot [128]
// int, and the row's score LSE [128] float (0 unless the gates come as raw scores).
constexpr uint32_t META_STAGE = 4 * 128 * 4;
constexpr uint32_t OFF_META = OFF_Q + NST * QTILE;
// Per O buffer and row: partial row index (or -1), 1/l, log2-sum-exp.
struct RowInfo {
  long long dst;
  float inv_l;
  float lse2;
};
constexpr uint32_t OFF_ROW = OFF_META + NST * META_STAGE;
// Epilogue staging: per epilogue warp its 32 rows of bf16 partials (256 bytes
// each, 16-byte chunks XOR-swizzled by row), so that the stores to global
// memory write whole rows (each warp store: two rows, four full 128-byte lines)
// instead of one 16-byte piece of 32 different rows.
constexpr uint32_t OFF_EPI = OFF_ROW + 2 * 128 * sizeof(RowInfo);
constexpr uint32_t EPI_WARP_BYTES = 32 * 256;
constexpr uint32_t OFF_BAR = OFF_EPI + 4 * EPI_WARP_BYTES;
constexpr uint32_t OFF_MISC = OFF_BAR + 256;
constexpr uint32_t SMEM_BYTES = OFF_MISC + 64 + 1024;   // + alignment slack
constexpr uint32_t COL_S = 0, COL_O = 128, TMEM_COLS = 512;   // S/P buffer b at 64 b, O buffer b at 128 + 128 b

struct Params {
  const __nv_bfloat16* Q;
  const float* logG;         // log gates, or raw scores when gate_lse is set
  const float* gate_lse;     // null, or the LSE of each row's historical scores
  const int32_t* cnt;        // per-block lists (sas_lists.cu), indexed by the global (b, g)
  const int32_t* off;
  const int32_t* list;
  const int32_t* list_cap;
  __nv_bfloat16* oslot;      // [groups of the batch][T][Ks][G][D] normalised partial outputs
  float* lslot;              // [groups of the batch][T][Ks][G] their log2-sum-exp
  int32_t* status;
  int bg0;                   // first (b, g) of the batch
  int Hq, Hkv, T, NB, G, P, Ks;
  float scale_log2;
  uint64_t wait_ns;
};

struct Bars {
  uint64_t kv_full, pos_ready[NST], q_full[NST], st_free[NST], s_full[2], p_full[2], s_free[2], o_full[2],
      o_free[2], fin;
};

__global__ void __launch_bounds__(THREADS, 1)
    sas_fwd_gather_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                          const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars* bars = reinterpret_cast<Bars*>(smem + OFF_BAR);
  RowInfo* rowinfo = reinterpret_cast<RowInfo*>(smem + OFF_ROW);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_MISC);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // Group-major order: the CTAs of one (b, g) run together, so the group's Q
  // rows (gathered about K times each) and K/V stay in L2. Within a group, small
  // j carry the longest row lists and start first.
  const int bgl = blockIdx.x / p.NB;   // (b, g) within the batch
  const int j = blockIdx.x % p.NB;
  const int bg = p.bg0 + bgl;
  const int b = bg / p.Hkv, g = bg % p.Hkv;
  const int PP = p.P, G = p.G;
  const int rows_used = G * PP;
  const int own_n = min(kBlock, p.T - j * kBlock);
  const int sel_n = min(p.cnt[(long long)bg * p.NB + j], p.list_cap[(long long)bg * p.NB + j]);
  const int total = own_n + sel_n;
  const int n_tiles = (total + PP - 1) / PP;
  const int32_t* lst = p.list + p.off[(long long)bg * p.NB + j];
  int32_t* status = p.status;
  const uint64_t wait_ns = p.wait_ns;

  if (warp == MMA_WARP) tmem_alloc(tmem_slot, TMEM_COLS);
  if (tid == 0) {
    mbar_init(&bars->kv_full, 1);
    for (int i = 0; i < NST; ++i) {
      mbar_init(&bars->pos_ready[i], 1);
      mbar_init(&bars->q_full[i], 1 + N_LOADER_WARPS);   // control (gates, slots) + loader warps (rows)
      mbar_init(&bars->st_free[i], 4);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->s_full[i], 1);
      mbar_init(&bars->p_full[i], 4);
      mbar_init(&bars->s_free[i], 1);
      mbar_init(&bars->o_full[i], 1);
      mbar_init(&bars->o_free[i], 4);
    }
    mbar_init(&bars->fin, 1);
    fence_barrier_init();
  }
  if (rows_used < 128) {   // rows never gathered stay zero
    const int per = (128 - rows_used) * 8;
    for (int i = tid; i < per * 2 * NST; i += THREADS) {
      const int stage = i / (2 * per), half = (i / per) & 1, rem = i % per;
      *reinterpret_cast<uint4*>(smem + OFF_Q + stage * QTILE + half * HALF128 + (rows_used + rem / 8) * 128 +
                                (rem % 8) * 16) = make_uint4(0, 0, 0, 0);
    }
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t s_base = smem_u32(smem);

  if (warp == CTRL_WARP) {
    // ------------------------------------------------------------------ control
    if (lane == 0) {
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      mbar_expect_tx(&bars->kv_full, 4 * KV_HALF);
      tma_load_3d(smem + OFF_K, &tmK, &bars->kv_full, 0, j * kBlock, bg);
      tma_load_3d(smem + OFF_K + KV_HALF, &tmK, &bars->kv_full, 64, j * kBlock, bg);
      tma_load_3d(smem + OFF_V, &tmV, &bars->kv_full, 0, j * kBlock, bg);
      tma_load_3d(smem + OFF_V + KV_HALF, &tmV, &bars->kv_full, 64, j * kBlock, bg);
    }
    // Entries (position | slot << kEntrySlotShift, -1 past the end) of tile i:
    // own positions first, then the list. The next tile's entries are loaded
    // while the current one is published, so the list's latency is not paid per tile.
    auto load_entries = [&](int i, int (&e)[4]) {
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int idx = i * PP + lane + 32 * u;
        e[u] = -1;
        if (lane + 32 * u < PP && idx < total) e[u] = idx < own_n ? j * kBlock + idx : lst[idx - own_n];
      }
    };
    int cur[4], nxt[4] = {-1, -1, -1, -1};
    load_entries(0, cur);
    for (int i = 0; i < n_tiles; ++i) {
      const int st = i % NST;
      if (i + 1 < n_tiles) load_entries(i + 1, nxt);
      bool ok = true;
      if (i >= NST) ok = mbar_wait(&bars->st_free[st], ((i / NST) - 1) & 1, status, wait_ns);
      if (!__all_sync(0xffffffffu, ok)) break;
      int* pos = reinterpret_cast<int*>(smem + OFF_META + st * META_STAGE);
      int* slot = pos + 256;
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (lane + 32 * u < PP) {
          pos[lane + 32 * u] = cur[u] >= 0 ? (cur[u] & kEntryPosMask) : -1;
          slot[lane + 32 * u] = cur[u] >= 0 ? (cur[u] >> kEntrySlotShift) : 0;
        }
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&bars->pos_ready[st]);
        mbar_arrive(&bars->q_full[st]);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) cur[u] = nxt[u];
    }
    if (lane == 0) mbar_wait_drain(&bars->kv_full, 0);
  } else if (warp >= LOADER_WARP0) {
    // ------------------------------------------------------------------ loaders: Q row gathers
    const int lt = tid - LOADER_WARP0 * 32;
    constexpr int NL = N_LOADER_WARPS * 32;
    const int per_pos = 16 * G;   // 16-byte pieces of a position's G rows
    const char* qbase = reinterpret_cast<const char*>(p.Q) + (long long)(b * p.Hq + g * G) * p.T * (D * 2);
    // Pieces ordered (position, head, 16-byte chunk), piece lt + k * NL for this
    // thread, so consecutive lanes copy consecutive bytes of one 256-byte row. The
    // map from a piece to its tile position, shared-memory offset and source
    // offset (head row, chunk) is the same for every tile: it is taken once, and
    // a tile then only reads its positions.
    constexpr int MAXP = (128 * 16 + NL - 1) / NL;   // G * P <= 128 rows of 16 pieces
    const int n_pieces = PP * per_pos;
    int pk_pp[MAXP];
    uint32_t pk_dst[MAXP], pk_src[MAXP];
#pragma unroll
    for (int k = 0; k < MAXP; ++k) {
      const int piece = lt + k * NL;
      const int pp = piece < n_pieces ? piece / per_pos : 0;
      const int rem = piece < n_pieces ? piece - pp * per_pos : 0;
      const int hh = rem >> 4, c16 = rem & 15;
      pk_pp[k] = piece < n_pieces ? pp : -1;
      pk_dst[k] = (uint32_t)(c16 >> 3) * HALF128 + sw128_offset((uint32_t)(hh * PP + pp), (uint32_t)(c16 & 7));
      pk_src[k] = (uint32_t)hh * (uint32_t)p.T * (D * 2) + (uint32_t)c16 * 16;   // < 2^31: G <= 16, T < 2^18
    }
    // Tiles are signalled in order as they land. A tile's copies are one cp.async
    // group per thread, so `issued - signalled` groups are in flight; waiting for
    // all but the newest n - 1 of them lands the oldest.
    int issued = 0, signalled = 0;
    auto signal_oldest = [&]() {
      const int n = issued - signalled;
      if (n >= 4)
        cp_async_wait_group<3>();
      else if (n == 3)
        cp_async_wait_group<2>();
      else if (n == 2)
        cp_async_wait_group<1>();
      else
        cp_async_wait_group<0>();
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->q_full[signalled % NST]);
      ++signalled;
    };
    for (int i = 0; i < n_tiles; ++i) {
      const int st = i % NST;
      bool ok = true;
      if (i >= NST) {
        // Until stage st is free again, signal the tiles in flight as they land:
        // the consumer of the stage waits on one of them.
        const uint32_t par = ((i / NST) - 1) & 1;
        while (true) {
          bool free_now = lane == 0 ? mbar_test_wait(&bars->st_free[st], par) : false;
          free_now = __shfl_sync(0xffffffffu, free_now, 0);
          if (free_now) break;
          if (issued > signalled) {
            signal_oldest();
            continue;
          }
          ok = mbar_wait(&bars->st_free[st], par, status, wait_ns);
          break;
        }
      }
      if (ok) ok = mbar_wait(&bars->pos_ready[st], (i / NST) & 1, status, wait_ns);
      if (!__all_sync(0xffffffffu, ok)) break;
      const int* pos = reinterpret_cast<const int*>(smem + OFF_META + st * META_STAGE);
      float* gate = reinterpret_cast<float*>(smem + OFF_META + st * META_STAGE) + 128;
      float* glse = gate + 256;
      const uint32_t qd = s_base + OFF_Q + st * QTILE;
      // The gate of block j for each selecting position (0 for own positions and
      // empty slots), with its row's score LSE when the gates come as raw scores,
      // copied in the same group as the rows.
      for (int pp = lt; pp < PP; pp += NL) {
        const int t = pos[pp];
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
      }
#pragma unroll
      for (int k = 0; k < MAXP; ++k) {
        if (pk_pp[k] < 0) continue;
        const int t = pos[pk_pp[k]];
        if (t < 0) continue;
        cp_async16(qd + pk_dst[k], qbase + pk_src[k] + (long long)t * (D * 2));
      }
      cp_async_commit();
      issued = i + 1;
      // At most LAG tiles in flight beyond the oldest: the gathers of several tiles overlap.
      if (issued - signalled > LAG) signal_oldest();
    }
    cp_async_wait_all();   // also after a failed wait: no copy may outlive the CTA
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0)
      for (int k = signalled; k < issued; ++k) mbar_arrive(&bars->q_full[k % NST]);
  } else if (warp == MMA_WARP) {
    // ------------------------------------------------------------------ MMA issuer
    // A polling state machine: S of the next tile and P V of the oldest tile are
    // issued as soon as their inputs are ready, in whichever order.
    if (lane == 0) {
      const uint32_t idesc_s = make_idesc_bf16(128, 64, 0, 0);    // rows x keys, K = features
      const uint32_t idesc_pv = make_idesc_bf16(128, D, 0, 1);    // rows x features, K = keys
      // Shared-memory descriptors: the address field is the byte address / 16, so
      // an operand at base + off (off a multiple of 16, inside the 256 KiB the
      // field spans) has descriptor desc(base) + off / 16. The bases are taken
      // once; each MMA adds a constant.
      const uint64_t d_q = make_sdesc(s_base + OFF_Q, 16, 1024);
      const uint64_t d_k = make_sdesc(s_base + OFF_K, 16, 1024);
      const uint64_t d_v = make_sdesc(s_base + OFF_V, KV_HALF, 1024);
      bool ok = mbar_wait(&bars->kv_full, 0, status, wait_ns);
      int ns = 0, np = 0;
      uint64_t t_last = global_ns();
      uint32_t spins = 0;
      while (ok && np < n_tiles) {
        bool prog = false;
        if (ns < n_tiles && ns < np + 2) {
          const int st = ns % NST, sb = ns & 1;
          if (mbar_test_wait(&bars->q_full[st], (ns / NST) & 1) &&
              (ns < 2 || mbar_test_wait(&bars->s_free[sb], ((ns - 2) >> 1) & 1))) {
            tc_fence_after();
            const uint64_t qs = (uint64_t)(st * QTILE) >> 4;   // this stage's offset in descriptor units
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
              const uint32_t half = ks >> 2, koff = (ks & 3) * 32;
              umma_ss(tmem + COL_S + 64 * sb, d_q + qs + ((half * HALF128 + koff) >> 4),
                      d_k + ((half * KV_HALF + koff) >> 4), idesc_s, ks > 0 ? 1u : 0u);
            }
            umma_commit(&bars->s_full[sb]);
            ++ns;
            prog = true;
          }
        }
        if (np < ns) {
          const int pb = np & 1;
          if (mbar_test_wait(&bars->p_full[pb], (np >> 1) & 1) &&
              (np < 2 || mbar_test_wait(&bars->o_free[pb], ((np - 2) >> 1) & 1))) {
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {   // K = 64 keys, 16 per MMA; A = P (bf16 pairs) in TMEM
              umma_ts(tmem + COL_O + 128 * pb, tmem + COL_S + 64 * pb + ks * 8, d_v + ((ks * 2048) >> 4), idesc_pv,
                      ks > 0 ? 1u : 0u);
            }
            umma_commit(&bars->o_full[pb]);
            umma_commit(&bars->s_free[pb]);
            ++np;
            prog = true;
          }
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
      umma_commit(&bars->fin);   // every MMA issued above completes before TMEM is released
      mbar_wait_drain(&bars->fin, 0);
    }
  } else if (warp >= EPI_WARP0) {
    // ------------------------------------------------------------------ epilogue (warps 4-7)
    const int quarter = warp - EPI_WARP0;
    const int r = quarter * 32 + lane;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    uint8_t* stage = smem + OFF_EPI + quarter * EPI_WARP_BYTES;
    for (int i = 0; i < n_tiles; ++i) {
      const int ob = i & 1;
      if (!warp_wait(&bars->p_full[ob], (i >> 1) & 1, status, wait_ns)) break;   // row info written
      if (!warp_wait(&bars->o_full[ob], (i >> 1) & 1, status, wait_ns)) break;
      tc_fence_after();
      const RowInfo info = rowinfo[ob * 128 + r];
      // O_j / l of this lane's row as bf16 into its staging row.
#pragma unroll 1
      for (int ch = 0; ch < D / 32; ch += 2) {   // two 32-column chunks per TMEM round trip
        uint32_t v[2][32];
        tmem_ld32(tmem + lane_base + COL_O + 128 * ob + 32 * ch, v[0]);
        tmem_ld32(tmem + lane_base + COL_O + 128 * ob + 32 * ch + 32, v[1]);
        tmem_wait_ld();
#pragma unroll
        for (int c2 = 0; c2 < 2; ++c2) {
          uint32_t w[16];
#pragma unroll
          for (int k = 0; k < 16; ++k)
            w[k] = pack_bf16(__uint_as_float(v[c2][2 * k]) * info.inv_l, __uint_as_float(v[c2][2 * k + 1]) * info.inv_l);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int cc = 4 * (ch + c2) + k;   // 16-byte chunk of the 256-byte row
            *reinterpret_cast<uint4*>(stage + lane * 256 + ((cc ^ (lane & 15)) << 4)) =
                make_uint4(w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
          }
        }
      }
      // The O buffer and its row info are free once TMEM is read: the stores
      // below use this warp's staging rows and registers only.
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->o_free[ob]);
      // Whole rows out: lanes 0-15 store row 2m, lanes 16-31 row 2m+1 (the
      // destination of row rr is held by lane rr).
      const int dlo = (int)(info.dst & 0xffffffffll), dhi = (int)(info.dst >> 32);
#pragma unroll 4
      for (int m = 0; m < 16; ++m) {
        const int rr = 2 * m + (lane >> 4), cc = lane & 15;
        const long long d = ((long long)__shfl_sync(0xffffffffu, dhi, rr) << 32) |
                            (uint32_t)__shfl_sync(0xffffffffu, dlo, rr);
        if (d >= 0) {
          const uint4 val = *reinterpret_cast<const uint4*>(stage + rr * 256 + ((cc ^ (rr & 15)) << 4));
          *reinterpret_cast<uint4*>(p.oslot + d * D + cc * 8) = val;
        }
      }
      if (info.dst >= 0) p.lslot[info.dst] = info.lse2;
      __syncwarp();   // the staging rows are rewritten by the next tile
    }
  } else {
    // ------------------------------------------------------------------ softmax (warps 0-3)
    const int r = tid;
    const int hh = r / PP, pp = r % PP;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    for (int i = 0; i < n_tiles; ++i) {
      const int st = i % NST, sb = i & 1;
      // The tile's metadata is published by q_full (waited here directly, not
      // only through the MMA thread), its S by s_full.
      if (!warp_wait(&bars->q_full[st], (i / NST) & 1, status, wait_ns)) break;
      if (!warp_wait(&bars->s_full[sb], (i >> 1) & 1, status, wait_ns)) break;
      tc_fence_after();
      const int* pos = reinterpret_cast<const int*>(smem + OFF_META + st * META_STAGE);
      int t = -1, sl = 0;
      float bias2 = 0.f;
      if (r < rows_used) {
        t = pos[pp];
        // log g = s - LSE(s) in fp32 (bit-identical to the normalised gate), then log2 units
        bias2 = (reinterpret_cast<const float*>(pos + 128)[pp] - reinterpret_cast<const float*>(pos + 384)[pp]) *
                kLog2e;
        sl = pos[256 + pp];
      }
      uint32_t sr[2][32];
      tmem_ld32(tmem + lane_base + COL_S + 64 * sb, sr[0]);
      tmem_ld32(tmem + lane_base + COL_S + 64 * sb + 32, sr[1]);
      tmem_wait_ld();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->st_free[st]);   // S is complete: the Q stage and its metadata are free
      const bool valid = t >= 0;
      const int lim = (valid && t / kBlock == j) ? t - j * kBlock : 63;   // causal limit in the own block
      float x[64];
      float mx = -INFINITY;
#pragma unroll
      for (int k = 0; k < 64; ++k) {
        x[k] = (valid && k <= lim) ? fmaf(__uint_as_float(sr[k >> 5][k & 31]), p.scale_log2, bias2) : -INFINITY;
        mx = fmaxf(mx, x[k]);
      }
      const float m_ref = (mx == -INFINITY) ? 0.f : mx;
      uint32_t pk[32];
      float l = 0.f;
#pragma unroll
      for (int k = 0; k < 32; ++k) {
        const float a0 = ex2(x[2 * k] - m_ref), a1 = ex2(x[2 * k + 1] - m_ref);
        l += a0 + a1;
        pk[k] = pack_bf16(a0, a1);
      }
      tmem_st32(tmem + lane_base + COL_S + 64 * sb, pk);   // P over the first half of its S buffer
      tmem_wait_st();
      // Row info of O buffer sb: free once the epilogue of tile i-2 has read it.
      if (i >= 2 && !warp_wait(&bars->o_free[sb], ((i - 2) >> 1) & 1, status, wait_ns)) break;
      RowInfo info;
      info.dst = valid ? (((long long)bgl * p.T + t) * p.Ks + sl) * G + hh : -1ll;
      info.inv_l = l > 0.f ? 1.f / l : 0.f;
      info.lse2 = l > 0.f ? m_ref + __log2f(l) : -INFINITY;
      rowinfo[sb * 128 + r] = info;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->p_full[sb]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

// Combines the slots of each position: one warp per (b, g, t), all G heads. A
// slot holds G rows of 128 bf16 (G * 256 contiguous bytes): lane l owns the
// 16-byte chunks l, l + 32, ... (KC of them, KC = ceil(G / 2)) and folds them
// over the slots with the weights exp2(lse_s - LSE) of their head. n = 1 +
// nsel[t] slots: slot 0 (own block) and the selected blocks.
// The kernel streams the partials once from HBM, so what matters is the number
// of loads in flight: the row's n * G log-sum-exps come in one coalesced pass
// into shared memory, where the per-head LSE is taken and each entry turned
// into its weight, while the first batch of slot loads is in flight.
constexpr int kMergeLseCap = 1024;   // Ks * G of the rows the merge takes
template <int KC>
__global__ void __launch_bounds__(256, 2) merge_kernel(const __nv_bfloat16* __restrict__ oslot,
                                                    const float* __restrict__ lslot,
                                                    const int32_t* __restrict__ nsel, __nv_bfloat16* __restrict__ O,
                                                    float* __restrict__ LSE, int bg0, long long n_rows, int T, int Ks,
                                                    int G, int Hq, int Hkv) {
  __shared__ float lse_sh[8][16];
  __shared__ float ls_sh[8][kMergeLseCap];
  const int wid = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long w = (long long)blockIdx.x * 8 + wid;
  if (w >= n_rows) return;
  const int t = (int)(w % T);
  const long long bgl = w / T;
  const long long bg = bg0 + bgl;
  const long long b = bg / Hkv, g = bg % Hkv;
  const int n = 1 + min(nsel[bg * T + t], Ks - 1);
  const long long row0 = (bgl * T + t) * Ks;   // first slot of the row
  const float* ls = lslot + row0 * G;          // [slot][head]
  const int n_chunks = 16 * G;
  const uint4* os = reinterpret_cast<const uint4*>(oslot + row0 * G * 128);   // slot s: G * 16 chunks
  constexpr int U = KC <= 4 ? 4 : 2;   // slots per batch of loads
  uint4 v[U][KC];
  // First batch of slot loads, in flight during the log-sum-exp reduction.
#pragma unroll
  for (int u = 0; u < U; ++u)
#pragma unroll
    for (int k = 0; k < KC; ++k) {
      const int c = lane + 32 * k;
      v[u][k] = (u < n && c < n_chunks) ? os[(long long)u * n_chunks + c] : make_uint4(0u, 0u, 0u, 0u);
    }
  float* lsw = ls_sh[wid];
  for (int e = lane; e < n * G; e += 32) lsw[e] = ls[e];
  __syncwarp();
  for (int hh = 0; hh < G; ++hh) {
    float M = -INFINITY;
    for (int s = lane; s < n; s += 32) M = fmaxf(M, lsw[s * G + hh]);
#pragma unroll
    for (int o = 16; o; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float L = 0.f;
    if (M != -INFINITY)
      for (int s = lane; s < n; s += 32) L += ex2(lsw[s * G + hh] - M);
#pragma unroll
    for (int o = 16; o; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
    // No finite partial cannot happen for valid inputs (the own block holds key t).
    const float lse2 = (M == -INFINITY) ? -INFINITY : M + __log2f(L);
    if (lane == 0) {
      lse_sh[wid][hh] = lse2;
      LSE[(b * Hq + g * G + hh) * T + t] = lse2 * kLn2;
    }
  }
  __syncwarp();
  // Each slot's weight per head, exp2(lse_s - LSE), in place (0 for an empty partial).
  for (int e = lane; e < n * G; e += 32) {
    const float x = lsw[e];
    lsw[e] = x == -INFINITY ? 0.f : ex2(x - lse_sh[wid][e % G]);
  }
  __syncwarp();
  float acc[KC][8];
#pragma unroll
  for (int k = 0; k < KC; ++k)
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[k][e] = 0.f;
  for (int s0 = 0; s0 < n; s0 += U) {
    if (s0 > 0) {
#pragma unroll
      for (int u = 0; u < U; ++u)
#pragma unroll
        for (int k = 0; k < KC; ++k) {
          const int c = lane + 32 * k;
          v[u][k] = (s0 + u < n && c < n_chunks) ? os[(long long)(s0 + u) * n_chunks + c] : make_uint4(0u, 0u, 0u, 0u);
        }
    }
#pragma unroll
    for (int u = 0; u < U; ++u)
#pragma unroll
      for (int k = 0; k < KC; ++k) {
        const int c = lane + 32 * k;
        if (s0 + u >= n || c >= n_chunks) continue;
        const float wu = lsw[(s0 + u) * G + (c >> 4)];
        const uint32_t x[4] = {v[u][k].x, v[u][k].y, v[u][k].z, v[u][k].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          acc[k][2 * e] = fmaf(wu, __uint_as_float(x[e] << 16), acc[k][2 * e]);
          acc[k][2 * e + 1] = fmaf(wu, __uint_as_float(x[e] & 0xffff0000u), acc[k][2 * e + 1]);
        }
      }
  }
#pragma unroll
  for (int k = 0; k < KC; ++k) {
    const int c = lane + 32 * k;
    if (c >= n_chunks) continue;
    const int hh = c >> 4;
    uint4 o;
    o.x = pack_bf16(acc[k][0], acc[k][1]);
    o.y = pack_bf16(acc[k][2], acc[k][3]);
    o.z = pack_bf16(acc[k][4], acc[k][5]);
    o.w = pack_bf16(acc[k][6], acc[k][7]);
    *reinterpret_cast<uint4*>(O + ((b * Hq + g * G + hh) * T + t) * 128 + (c & 15) * 8) = o;
  }
}

// Partials of one (b, g) may take at most this many bytes of workspace; larger
// problems (long rows with large budgets) run the union forward instead.
constexpr size_t kSlotBudget = size_t(8) << 30;

int slots_per_row(int K, int NB) { return 1 + std::max(0, std::min(K - 1, NB)); }

size_t slot_bytes_per_group(int Hq, int Hkv, int T, int K) {
  const int G = Hq / Hkv;
  return (size_t)T * slots_per_row(K, T / kBlock) * G * (D * 2 + 4);
}

// Groups per batch: all of them when their partials fit the budget, else an
// even split into batches that do.
int groups_per_batch(int B, int Hq, int Hkv, int T, int K) {
  const long long nbg = (long long)B * Hkv;
  const size_t per = slot_bytes_per_group(Hq, Hkv, T, K);
  const long long fit = std::max<long long>(1, (long long)(kSlotBudget / per));
  const long long n_batches = (nbg + fit - 1) / fit;
  return (int)((nbg + n_batches - 1) / n_batches);
}

}  // namespace gfwd

bool fwd_gather_applies(int B, int Hq, int Hkv, int T, int K) {
  (void)B;
  return gfwd::slot_bytes_per_group(Hq, Hkv, T, K) <= gfwd::kSlotBudget &&
         gfwd::slots_per_row(K, T / kBlock) * (Hq / Hkv) <= gfwd::kMergeLseCap;
}

size_t fwd_gather_workspace_bytes(int B, int Hq, int Hkv, int T, int K) {
  using namespace gfwd;
  const int NB = T / kBlock;
  const long long nbg = (long long)B * Hkv;
  const int G = Hq / Hkv, Ks = slots_per_row(K, NB);
  const long long rows = (long long)groups_per_batch(B, Hq, Hkv, T, K) * T * Ks * G;
  auto a256 = [](size_t x) { return (x + 255) / 256 * 256; };
  return block_lists_bytes(nbg, T, NB, K) + a256((size_t)rows * D * 2) + a256((size_t)rows * 4);
}

cudaError_t launch_fwd_gather(const TcProblem& pb, int K, void* O, float* LSE, int32_t* status, uint8_t* scratch,
                              cudaStream_t st) {
  using namespace gfwd;
  const int NB = pb.NB;
  const long long nbg = (long long)pb.B * pb.Hkv;
  const int Ks = slots_per_row(K, NB);
  const int gpb = groups_per_batch(pb.B, pb.Hq, pb.Hkv, pb.T, K);
  auto a256 = [](size_t x) { return (x + 255) / 256 * 256; };
  const BlockLists L = carve_block_lists(scratch, nbg, pb.T, NB, K);
  size_t o = block_lists_bytes(nbg, pb.T, NB, K);
  const long long slot_rows = (long long)gpb * pb.T * Ks * pb.G;
  __nv_bfloat16* oslot = reinterpret_cast<__nv_bfloat16*>(scratch + o);
  o += a256((size_t)slot_rows * D * 2);
  float* lslot = reinterpret_cast<float*>(scratch + o);

  cudaError_t e =
      launch_block_lists(pb.logG, pb.gate_lse, pb.tau, pb.tau_idx, pb.sel, L, nbg, pb.T, NB, K, true, status, st);
  if (e != cudaSuccess) return e;
  const QTileShape qs = qtile_shape(pb.G, pb.T, NB);
  CUtensorMap tk, tv;
  if (!make_tmap_bf16_3d(&tk, pb.K, pb.d, pb.T, (uint64_t)nbg, 64) ||
      !make_tmap_bf16_3d(&tv, pb.V, pb.d, pb.T, (uint64_t)nbg, 64))
    return cudaErrorInvalidValue;
  Params prm;
  prm.Q = reinterpret_cast<const __nv_bfloat16*>(pb.Q);
  prm.logG = pb.logG;
  prm.gate_lse = pb.gate_lse;
  prm.cnt = L.cnt;
  prm.off = L.off;
  prm.list = L.list;
  prm.list_cap = L.cap;
  prm.oslot = oslot;
  prm.lslot = lslot;
  prm.status = status;
  prm.Hq = pb.Hq;
  prm.Hkv = pb.Hkv;
  prm.T = pb.T;
  prm.NB = NB;
  prm.G = pb.G;
  prm.P = qs.P;
  prm.Ks = Ks;
  prm.scale_log2 = pb.sm_scale * kLog2e;
  prm.wait_ns = wait_limit_ns();
  if ((e = cudaFuncSetAttribute(sas_fwd_gather_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES)) !=
      cudaSuccess)
    return e;
  for (long long bg0 = 0; bg0 < nbg; bg0 += gpb) {
    const int n_in = (int)std::min<long long>(gpb, nbg - bg0);
    prm.bg0 = (int)bg0;
    sas_fwd_gather_kernel<<<(unsigned)(n_in * NB), THREADS, SMEM_BYTES, st>>>(tk, tv, prm);
    count_launch();
    const long long n_rows = (long long)n_in * pb.T;
    const unsigned mgrid = (unsigned)((n_rows + 7) / 8);
    __nv_bfloat16* Ob = reinterpret_cast<__nv_bfloat16*>(O);
    if (pb.G <= 2)
      merge_kernel<1><<<mgrid, 256, 0, st>>>(oslot, lslot, L.nsel, Ob, LSE, (int)bg0, n_rows, pb.T, Ks, pb.G, pb.Hq, pb.Hkv);
    else if (pb.G <= 4)
      merge_kernel<2><<<mgrid, 256, 0, st>>>(oslot, lslot, L.nsel, Ob, LSE, (int)bg0, n_rows, pb.T, Ks, pb.G, pb.Hq, pb.Hkv);
    else if (pb.G <= 6)
      merge_kernel<3><<<mgrid, 256, 0, st>>>(oslot, lslot, L.nsel, Ob, LSE, (int)bg0, n_rows, pb.T, Ks, pb.G, pb.Hq, pb.Hkv);
    else if (pb.G <= 8)
      merge_kernel<4><<<mgrid, 256, 0, st>>>(oslot, lslot, L.nsel, Ob, LSE, (int)bg0, n_rows, pb.T, Ks, pb.G, pb.Hq, pb.Hkv);
    else
      merge_kernel<8><<<mgrid, 256, 0, st>>>(oslot, lslot, L.nsel, Ob, LSE, (int)bg0, n_rows, pb.T, Ks, pb.G, pb.Hq, pb.Hkv);
    count_launch();
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace sas
