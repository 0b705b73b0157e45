/*
 * sas.h - C ABI of the SAS gated block-sparse attention library for NVIDIA B200 (sm_100a).
 *
 * The operation is the one defined in "SAS: Simple Attention Sparsification via
 * End-to-End Optimization of Context Ranking" (arXiv 2609.13141), cited below as
 * "SAS paper":
 *
 *   * a selector score s[m] per historical context block becomes a gate
 *     g = softmax(s) over the historical blocks, used in log form
 *     (§4.1 eq. 4, §4.2 "Activation function" eq. 6);
 *   * each query keeps its current block B_0 (unit gate, causal) and the
 *     Top-(K-1) historical blocks, realised as a per-query threshold on the log
 *     gate (§4.3 "Kernel Design", Appendix E);
 *   * attention is softmax(q K_S^T + log g_S) V_S over the kept tokens
 *     (§4.3 eq. 9), with dQ/dK/dV and the block-level gate gradient in the
 *     backward pass (Appendix E "Backward pass"; Appendix D.1 eq. 5);
 *   * decoding selects Top-(K-1) historical blocks by score and runs ungated
 *     attention over them and the current block (§4.3 Algorithm 2; §5.1
 *     "Inference implementation"), from a contiguous or a paged KV cache;
 *   * around the path: the gradient with respect to the selector scores
 *     (Appendix D.3), the noisy "full*" selection (§4.1, Table 1), and packed
 *     sequences of documents (§5.1).
 *
 * Entry points: sas_gate_normalize, sas_select_threshold and their fused form
 * sas_gate_normalize_select (and _varlen for packed documents, _compact for
 * gates kept as scores + a row log-sum-exp), sas_select_noisy,
 * sas_fwd, sas_bwd, sas_gate_grad, sas_decode_fwd (and _paged, _static), the
 * workspace sizes, the device status word, sas_status_string, sas_version and
 * sas_launch_count.
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Blocks are `block` = 64 consecutive tokens. Query position t is in block
 *    c_t = t / 64; its historical blocks are m < c_t.
 *  - K (the budget) counts blocks and INCLUDES the current block: H = K - 1
 *    historical blocks are kept per query.
 *  - Grouped-query attention: Hq query heads, Hkv KV heads, G = Hq / Hkv. Query
 *    head h uses KV head g = h / G. Gates, thresholds and selections are per
 *    (batch, KV head, position) and shared by the G query heads of the group.
 *  - Layouts are dense row-major, innermost dimension last:
 *      Q, O, dO, dQ : [B, Hq, T, d]          K, V, dK, dV : [B, Hkv, T, d]
 *      s, logG, dLogG : [B, Hkv, T, NB] fp32  tau : [B, Hkv, T] fp32
 *      tau_idx : [B, Hkv, T] int32            LSE : [B, Hq, T] fp32 (natural log)
 *  - Pointers are DEVICE pointers unless stated otherwise. The caller owns every
 *    buffer, including the workspace; the library never allocates or frees
 *    device memory. All device pointers must be 16-byte aligned.
 *  - Every call is asynchronous on `stream` (a cudaStream_t passed as void*;
 *    NULL = the legacy default stream). Arguments are validated on the host
 *    before anything is launched; an invalid call returns an error and
 *    launches nothing.
 *  - Kernel-side failures (a bounded wait that expired, an index out of range) are
 *    recorded in a status word at the start of the workspace; read it with
 *    sas_device_status(). Once the word holds an error, every later bounded wait
 *    of the call gives up, so the outputs of that call are not defined; clear the
 *    word (sas_device_status_clear) before reusing the workspace.
 *  - sm_scale multiplies q.k only; the log gate is added unscaled.
 *  - The fp32 data type runs on a CUDA-core kernel; bf16 runs on tcgen05
 *    tensor-core kernels (fwd/bwd: d = 128).
 */
#ifndef SAS_B200_H
#define SAS_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SAS_API __attribute__((visibility("default")))
#else
#define SAS_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes returned by every call. */
typedef enum {
  SAS_OK = 0,
  SAS_ERR_INVALID_ARG = -1, /* bad pointer, size, alignment or combination of sizes */
  SAS_ERR_UNSUPPORTED = -2, /* valid, but not a shape/dtype this build implements */
  SAS_ERR_CUDA = -3,        /* a CUDA runtime call failed (e.g. a launch error) */
  SAS_ERR_TIMEOUT = -4,     /* a kernel's bounded wait expired (reported by sas_device_status) */
  SAS_ERR_WORKSPACE = -5    /* workspace missing or smaller than the *_workspace_size answer */
} sas_status;

/* Element types of Q/K/V/O/dO/dQ/dK/dV. */
typedef enum { SAS_DT_F32 = 0, SAS_DT_BF16 = 1 } sas_dtype;

/* Human-readable name of a status code. Never NULL. */
SAS_API const char* sas_status_string(int status);

/* Library ABI version (major * 100 + minor). */
SAS_API int sas_version(void);

/* Number of kernels this library has launched since it was loaded (all threads). */
SAS_API uint64_t sas_launch_count(void);

/*
 * sas_set_wait_limit_ns - limit (nanoseconds) of each bounded wait inside the
 * sas_fwd and sas_bwd tensor-core kernels launched after this call (process-wide;
 * 0 restores the default of 1 s). A wait that exceeds it records a timeout in the
 * workspace status word (sas_device_status) and the kernel winds down: it lets the
 * copies and MMAs it has issued finish, releases its tensor memory and returns,
 * leaving its outputs incomplete. Meant for testing the failure path; a limit of a
 * few microseconds makes the first wait of every CTA expire. Returns the previous
 * limit. Not synchronised with calls in flight on other host threads.
 */
SAS_API uint64_t sas_set_wait_limit_ns(uint64_t ns);

/*
 * sas_gate_normalize - softmax gate activation in log form.
 * SAS paper §4.1 eq. 4 (g = phi(s), g_0 = 1) with phi = softmax, §4.2 eq. 6:
 *   logG[b,g,t,m] = s[b,g,t,m] - log sum_{m' < c_t} exp(s[b,g,t,m'])   for m < c_t,
 *   logG[b,g,t,m] = -inf                                               for m >= c_t.
 * s, logG: [B, Hkv, T, NB] fp32 (may not alias). NB >= ceil(T / block).
 * block must be 64. Rows with c_t = 0 are all -inf.
 */
SAS_API int sas_gate_normalize(const float* s, float* logG, int B, int Hkv, int T, int NB, int block, void* stream);

/*
 * sas_select_threshold - Top-(K-1) historical blocks per query as a threshold.
 * SAS paper §4.3 "Kernel Design" and Appendix E: block m < c_t is selected iff
 *   logG[m] > tau  or  (logG[m] == tau and m <= tau_idx),
 * which keeps exactly min(K-1, c_t) blocks: the K-1 largest values, equal values
 * going to the lower block index (-0.0 equals +0.0). Rows with c_t <= K-1 keep
 * every historical block (tau = -inf, tau_idx = c_t - 1); rows that keep none
 * (c_t = 0 or K = 1) get tau = +inf, tau_idx = -1.
 * logG: [B,Hkv,T,NB] fp32, finite for m < c_t. tau: [B,Hkv,T] fp32.
 * tau_idx: [B,Hkv,T] int32. sel (nullable): [B,Hkv,T,K-1] int32, the selected
 * block indices in ascending order, padded with -1. K >= 1, block == 64.
 */
SAS_API int sas_select_threshold(const float* logG, float* tau, int32_t* tau_idx, int32_t* sel, int B, int Hkv, int T,
                         int NB, int block, int K, void* stream);

/*
 * sas_gate_normalize_select - sas_gate_normalize followed by sas_select_threshold
 * in one pass over s: logG, tau, tau_idx and sel are bit for bit the values the
 * two calls produce (same arithmetic and summation order), with s read once and
 * logG not read back. Arguments, layouts and errors are those of the two calls
 * (s and logG may not alias).
 */
SAS_API int sas_gate_normalize_select(const float* s, float* logG, float* tau, int32_t* tau_idx, int32_t* sel, int B,
                                      int Hkv, int T, int NB, int block, int K, void* stream);

/*
 * sas_gate_normalize_select_compact - sas_gate_normalize_select without the logG
 * tensor (SAS paper §4.2 eq. 6: log g = s - log sum exp over the historical
 * blocks; Appendix D.3). It writes, per (b, g, t), the log-sum-exp of the row's
 * historical scores,
 *   gate_lse[b,g,t] = log sum_{m < c_t} exp(s[b,g,t,m])     (-inf when c_t = 0),
 * and tau, tau_idx, sel exactly as sas_gate_normalize_select does (bit for bit):
 * the selection is taken on logG[m] = s[m] - gate_lse (one fp32 subtraction,
 * the value sas_gate_normalize writes). sas_fwd, sas_bwd and sas_gate_grad given
 * s in place of logG together with gate_lse rebuild the same gates, so a
 * training step reads s where it read logG and never writes the dense logG.
 * gate_lse: [B, Hkv, T] fp32. Other arguments as for sas_gate_normalize_select;
 * NB <= 1024 (else SAS_ERR_UNSUPPORTED).
 */
SAS_API int sas_gate_normalize_select_compact(const float* s, float* gate_lse, float* tau, int32_t* tau_idx,
                                              int32_t* sel, int B, int Hkv, int T, int NB, int block, int K,
                                              void* stream);

/*
 * sas_gate_normalize_select_varlen - sas_gate_normalize_select for a packed
 * sequence of documents (SAS paper §5.1: training on packed sequences). Document
 * i covers tokens cu_seqlens[i] .. cu_seqlens[i+1]-1 and blocks
 * cu_seqlens[i]/64 .. cu_seqlens[i+1]/64-1; it never sees another document. For
 * a row t of document i (c = t/64, c_i = cu_seqlens[i]/64) the gates are the
 * softmax of s over its own earlier blocks c_i .. c-1 (logG = -inf on every other
 * column) and the Top-(K-1) is taken among them (ties to the lower block); block
 * indices in tau_idx and sel are those of the packed sequence. A row keeping every
 * block of its document (c - c_i <= K-1) gets (-inf, c-1) in the first document
 * and, in later ones, (the least of its gates, the last block holding it), so that
 * the threshold keeps no block of an earlier document; a row keeping nothing gets
 * (+inf, -1). sas_fwd, sas_bwd and sas_gate_grad take these outputs as they are:
 * the attended set of every row lies inside its own document.
 * cu_seqlens: HOST int32 [n_docs + 1], 0 = cu[0] < cu[1] < ... < cu[n_docs] = T,
 * every entry a multiple of 64; 1 <= n_docs <= 256 (more: SAS_ERR_UNSUPPORTED).
 * Other arguments as for sas_gate_normalize_select; NB <= 1024 (else
 * SAS_ERR_UNSUPPORTED). The same packing applies to every (b, g).
 */
SAS_API int sas_gate_normalize_select_varlen(const float* s, float* logG, float* tau, int32_t* tau_idx, int32_t* sel,
                                             int B, int Hkv, int T, int NB, int block, int K,
                                             const int32_t* cu_seqlens, int n_docs, void* stream);

/*
 * sas_select_noisy - selection for the "full*" training scope (SAS paper §4.1,
 * Table 1 row 11: noise added to the selector scores before Top-K). Per (b, g, t)
 * with c = min(t / 64, NB) historical blocks:
 *   chosen = the K-1 largest of key[m] = logG[m] + noise[m] (an fp32 add) over
 *            m < c, ties to the lower block (every historical block when c <= K-1);
 *   logG_sel[m] = logG[m] for m in chosen, -inf otherwise;
 *   (tau, tau_idx) = the threshold of logG_sel, as sas_select_threshold would give
 *            it: the least kept gate (-0 written as +0) and the largest kept block
 *            holding it; (-inf, c-1) when c <= K-1; (+inf, -1) when nothing is kept.
 * sas_fwd / sas_bwd given (logG_sel, tau, tau_idx) attend exactly the chosen blocks
 * with the clean gates logG on them; the gradient they return for logG_sel is the
 * gradient for logG (zero off the chosen blocks), for sas_gate_grad with logG.
 * Blocks whose gate is -inf (other documents of a packed sequence, from
 * sas_gate_normalize_select_varlen) are never chosen; a row with fewer gated
 * blocks than K-1 keeps all of them, with (the least kept gate, the last block
 * holding it) as its threshold unless they are all its historical blocks.
 * logG, noise, logG_sel: [B,Hkv,T,NB] fp32 (logG_sel may alias neither input);
 * tau [B,Hkv,T] fp32; tau_idx [B,Hkv,T] int32; sel (nullable) [B,Hkv,T,K-1] int32,
 * the chosen blocks ascending, -1 padded. The caller draws the noise.
 * NB >= ceil(T / 64), NB <= 1024 (else SAS_ERR_UNSUPPORTED), block == 64, K >= 1.
 */
SAS_API int sas_select_noisy(const float* logG, const float* noise, float* logG_sel, float* tau, int32_t* tau_idx,
                             int32_t* sel, int B, int Hkv, int T, int NB, int block, int K, void* stream);

/*
 * sas_gate_grad - gradient with respect to the selector scores s through the
 * gate normalisation (SAS paper Appendix D.3, the softmax backward
 * ds_m = g_m (dg_m - sum_l g_l dg_l), with the gate gradient given in log form
 * dLogG_l = g_l dg_l as sas_bwd returns it, and g = exp(logG)):
 *   ds[b,g,t,m] = dLogG[b,g,t,m] - exp(logG[b,g,t,m]) * sum_{l < c_t} dLogG[b,g,t,l]  for m < c_t,
 *   ds[b,g,t,m] = 0                                                                   for m >= c_t.
 * logG (from sas_gate_normalize), dLogG, ds: [B,Hkv,T,NB] fp32; ds may not alias
 * either input. With gate_lse non-null (compact gates from
 * sas_gate_normalize_select_compact), `logG` holds the raw scores s and
 * logG[m] = s[m] - gate_lse[b,g,t] is rebuilt in fp32. NB >= ceil(T / block),
 * block == 64.
 */
SAS_API int sas_gate_grad(const float* logG, const float* gate_lse, const float* dLogG, float* ds, int B, int Hkv,
                          int T, int NB, int block, void* stream);

/*
 * Workspace sizes (bytes) for sas_fwd, sas_bwd and sas_decode_fwd with the given
 * sizes. The workspace is caller-owned device memory, at least 256-byte aligned,
 * and may be reused across calls on the same stream. Its first word is the
 * device status word.
 */
SAS_API int sas_fwd_workspace_size(int B, int Hq, int Hkv, int T, int d, int block, int K, int dtype,
                                   size_t* bytes);
SAS_API int sas_bwd_workspace_size(int B, int Hq, int Hkv, int T, int d, int block, int K, int dtype,
                               size_t* bytes);
SAS_API int sas_decode_workspace_size(int B, int Hq, int Hkv, int Lmax, int d, int block, int K, size_t* bytes);

/*
 * sas_fwd - gated block-sparse attention forward (SAS paper §4.3 eq. 9, Appendix E
 * Algorithm 3 "Forward Pass"):
 *   O[b,h,t]   = sum_i softmax_i(z) V[b,g,i],   z_i = sm_scale q.k_i + bias(t, i),
 *   LSE[b,h,t] = log sum_i exp(z_i),
 * with bias = 0 for keys of the current block with i <= t, logG[b,g,t,m] for keys
 * of a selected historical block m (selection as in sas_select_threshold), and
 * -inf for every other key.
 * Q [B,Hq,T,d], K/V [B,Hkv,T,d] of `dtype`; logG [B,Hkv,T,NB], tau, tau_idx as
 * produced by the two calls above (any values obeying their contract work).
 * gate_lse: null, or (compact gates, sas_gate_normalize_select_compact) the
 * [B,Hkv,T] log-sum-exp of each row's historical scores, with the raw scores s
 * passed as `logG`: the gate is then s[m] - gate_lse[b,g,t] in fp32, bit for bit
 * the normalised gate.
 * sel: null, or the index list the selection call wrote with the same tau and
 * tau_idx ([B,Hkv,T,Kbudget-1] int32, each row's selected blocks ascending, -1
 * padded). The bf16 kernels then build their per-block row lists from it (4 bytes
 * per selected block) instead of thresholding each row's gates again; the
 * attended set and the results are the same. An entry that is not an earlier
 * block of its row is never used to index anything and is reported as a
 * device-side bounds error (the call's outputs are then not defined).
 * O [B,Hq,T,d] of `dtype`; LSE [B,Hq,T] fp32. T % 64 == 0, NB == T / 64,
 * Hq % Hkv == 0, d in {64, 128} (fp32) or d == 128 (bf16).
 * Kbudget: the budget K given to the selection (the threshold keeps at most K-1
 * historical blocks per row; a threshold that keeps more is reported as a
 * device-side bounds error, and the call's outputs are then not defined). For bf16 the
 * workspace holds per-block row lists and one partial output per (position,
 * attended block), about T * K * Hq/Hkv KiB per (b, g), processed in batches of
 * (b, g) of at most 8 GiB of partials; when one (b, g) alone needs more, or a
 * row has more than 1024 partials (min(K, NB + 1) x Hq/Hkv), the call runs a
 * q-tile kernel over the union of each tile's blocks instead and the workspace is
 * small.
 * ws: workspace of sas_fwd_workspace_size bytes (same K).
 */
SAS_API int sas_fwd(const void* Q, const void* K, const void* V, int dtype, const float* logG, const float* gate_lse,
                    const float* tau, const int32_t* tau_idx, const int32_t* sel, void* O, float* LSE, int B, int Hq,
                    int Hkv, int T, int d, int block, int Kbudget, float sm_scale, void* ws, size_t ws_bytes,
                    void* stream);

/*
 * sas_bwd - gradients of a scalar loss through sas_fwd (SAS paper Appendix E
 * "Backward pass", Algorithm 4; gate gradient per Appendix D.1 eq. 5 / D.3):
 *   P = exp(z - LSE), Delta = rowsum(O * dO), dS = P * (dO V^T - Delta),
 *   dQ = sm_scale dS K,  dK = sm_scale sum_{h in g} dS^T Q,  dV = sum_{h in g} P^T dO,
 *   dLogG[b,g,t,m] = sum_{h in g} sum_{i in block m} dS[h,t,i] for selected m, 0 otherwise.
 * Inputs as for sas_fwd (gate_lse and sel included) plus O (the forward output),
 * dO and LSE (the forward's).
 * Outputs dQ [B,Hq,T,d], dK/dV [B,Hkv,T,d] of `dtype`; dLogG [B,Hkv,T,NB] fp32
 * (fully written: zero outside the selection). Kbudget: the budget K given to
 * sas_select_threshold (the threshold keeps at most K-1 historical blocks per row;
 * internal per-block row lists are sized by it; a threshold that keeps more is
 * reported as a device-side bounds error, and the outputs are then not defined).
 * ws: sas_bwd_workspace_size bytes
 * (for bf16 it holds an fp32 dQ accumulator and the per-block row lists).
 */
SAS_API int sas_bwd(const void* Q, const void* K, const void* V, const void* O, const void* dO, int dtype,
                    const float* logG, const float* gate_lse, const float* tau, const int32_t* tau_idx,
                    const int32_t* sel, const float* LSE, void* dQ, void* dK, void* dV, float* dLogG, int B, int Hq,
                    int Hkv, int T, int d, int block, int Kbudget, float sm_scale, void* ws, size_t ws_bytes,
                    void* stream);

/*
 * sas_decode_fwd - one sparse decode step per sequence (SAS paper §4.3
 * Algorithm 2; §5.1 "Inference implementation", §6.3):
 *   L = seqlen[b] (the new token is position L-1), c = (L-1) / 64;
 *   I = Top-(K-1) of blocks 0..c-1 by s[b,g,:] (ties to the lower index);
 *   o[b,h] = softmax(sm_scale q K_S^T + bias) V_S over S = block c (positions
 *   c*64 .. L-1) and the blocks in I; bias = 0 (ungated, Algorithm 2) or, with
 *   apply_log_gate != 0, s[b,g,m] - log sum_{m'<c} exp(s[b,g,m']) on block m in I.
 * q [B,Hq,d], Kc/Vc [B,Hkv,Lmax,d] of `dtype` (the KV cache; the new token's
 * key/value already at position L-1); seqlen [B] int32 DEVICE, 1 <= L <= Lmax;
 * s [B,Hkv,NBmax] fp32 with NBmax >= ceil(Lmax/64); o [B,Hq,d] of `dtype`;
 * sel_out (nullable) [B,Hkv,K-1] int32 receives I in ascending order, -1 padded.
 * d == 128, 1 <= K <= 64. ws: sas_decode_workspace_size bytes. A seqlen
 * outside 1..Lmax is reported as a device-side bounds error (sas_device_status).
 */
SAS_API int sas_decode_fwd(const void* q, const void* Kc, const void* Vc, int dtype, const int32_t* seqlen, const float* s,
                   int K, int apply_log_gate, void* o, int32_t* sel_out, int B, int Hq, int Hkv, int Lmax, int NBmax,
                   int d, int block, float sm_scale, void* ws, size_t ws_bytes, void* stream);

/*
 * sas_decode_fwd_paged - sas_decode_fwd over a paged KV cache (SAS paper §5.1
 * "Inference implementation": a paged cache, only the selected KV blocks
 * gathered). The computation is that of sas_decode_fwd on the logical cache in
 * which token p of sequence b is row p % 64 of page page_table[b, p / 64].
 * Kp/Vp [num_pages, Hkv, 64, d] bf16: one page holds one 64-token block of every
 * KV head (the head's 64 rows contiguous). page_table [B, max_pages] int32
 * DEVICE; entries of blocks 0..(seqlen[b]-1)/64 must lie in 0..num_pages-1 (an
 * entry outside is reported as a device-side bounds error and no copy is issued
 * for its block; o is then not defined); entries past a sequence's last block are
 * never read. Pages may be
 * shared between sequences. seqlen [B] int32 DEVICE, 1 <= L <= max_pages * 64.
 * s [B,Hkv,NBmax] fp32 with NBmax >= max_pages. Other arguments, the workspace
 * (sas_decode_workspace_size with Lmax = max_pages * 64) and errors as for
 * sas_decode_fwd; dtype must be SAS_DT_BF16 (fp32 returns SAS_ERR_UNSUPPORTED).
 * Captures into a CUDA graph (no allocation, no host synchronisation).
 */
SAS_API int sas_decode_fwd_paged(const void* q, const void* Kp, const void* Vp, int dtype, const int32_t* page_table,
                                 int max_pages, int num_pages, const int32_t* seqlen, const float* s, int K,
                                 int apply_log_gate, void* o, int32_t* sel_out, int B, int Hq, int Hkv, int NBmax,
                                 int d, int block, float sm_scale, void* ws, size_t ws_bytes, void* stream);

/*
 * sas_decode_fwd_static - sas_decode_fwd without a workspace argument. It has no
 * counterpart in the SAS paper; it exists for callers that cannot allocate device
 * memory themselves: a plugin whose host framework owns every device buffer and
 * hands it only inputs and outputs, or a latency-critical decode loop that must
 * not call cudaMalloc (which can synchronise the device) between steps.
 *
 * Arguments, layouts, results and errors are those of sas_decode_fwd, minus
 * ws/ws_bytes. The scratch memory sas_decode_fwd would take from the workspace
 * lives instead in one static 8 MiB device array inside the library:
 *  - every GPU that loads the library holds those 8 MiB until the process exits;
 *  - a problem whose sas_decode_workspace_size exceeds 8 MiB (8388608 bytes) is
 *    rejected with SAS_ERR_WORKSPACE before anything is launched;
 *  - the call allocates nothing (no cudaMalloc, cudaFree or allocating library
 *    routine); it clears the parts of the array that must start at zero on
 *    every call, with asynchronous memsets on `stream`;
 *  - all calls on a device share the array, so calls whose kernels overlap on the
 *    GPU (different streams, or different host threads) race on it and give
 *    wrong results: serialise them;
 *  - the first call on each device looks up the array's device address (with that
 *    device current) and caches it per CUDA context (a device reset or a re-created
 *    primary context triggers a new lookup); make that first call before any stream
 *    capture;
 *  - the array's status word is cleared at the start of every call; read it after
 *    a call with sas_decode_static_status().
 */
SAS_API int sas_decode_fwd_static(const void* q, const void* Kc, const void* Vc, int dtype, const int32_t* seqlen,
                                  const float* s, int K, int apply_log_gate, void* o, int32_t* sel_out, int B,
                                  int Hq, int Hkv, int Lmax, int NBmax, int d, int block, float sm_scale,
                                  void* stream);

/*
 * sas_decode_static_status - the device status word of the last sas_decode_fwd_static
 * call on the current device: synchronises `stream`, copies the word of the static
 * array to *status_out (0 = no kernel-side error; a seqlen outside 1..Lmax is a
 * bounds error) and returns SAS_ERR_TIMEOUT if it is non-zero, else SAS_OK. Like
 * the entry point it reads, it has no counterpart in the SAS paper and allocates
 * nothing.
 */
SAS_API int sas_decode_static_status(void* stream, int32_t* status_out);

/*
 * sas_device_status - read the device status word of a workspace used by
 * sas_fwd/sas_bwd/sas_decode_fwd. Synchronises `stream`, copies the word to
 * *status_out (0 = no kernel-side error) and returns SAS_ERR_TIMEOUT if a bounded
 * wait expired, else SAS_OK. sas_device_status_clear() zeroes it (asynchronously).
 */
SAS_API int sas_device_status(const void* ws, void* stream, int32_t* status_out);
SAS_API int sas_device_status_clear(void* ws, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SAS_B200_H */
