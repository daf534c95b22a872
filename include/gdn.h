/*
 * gdn.h -- C ABI of libgdn.so: the Gated DeltaNet (gated delta rule) hot path
 * on one NVIDIA B200 (sm_100a).
 *
 * Per (sequence, value head) the library computes the gated delta rule
 *     S_t = exp(g_t) * S_{t-1} * (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,
 *     o_t = scale * S_t q_t,
 * with the state held in f32 as H = S^T, row-major [d_k][d_v].
 *
 * Conventions shared by every entry point
 *   - All pointers are DEVICE pointers unless stated; the caller owns every
 *     buffer.  No entry point allocates, frees or synchronises: work is queued
 *     on `stream` (a cudaStream_t; 0 = the legacy default stream) and the call
 *     returns.
 *   - bf16 tensors are passed as `uint16_t*` holding bf16 bit patterns.
 *   - Strides are in ELEMENTS between consecutive tokens (rows).
 *   - v-head h reads k-head h / (H_v / H_k) (heads grouped contiguously, the
 *     grouping ba_gates_slot uses on the BA page).
 *   - Every call returns GDN_OK or a GDN_ERR_* code.  On an error nothing is
 *     launched and gdn_last_error() names the guard that refused (thread-local
 *     string, valid until the next call on the same thread).
 *   - Device-side problems never trap: verify/fold report them in bit 1
 *     (GDN_FLAG_ERROR) of the engaged word.
 *
 * Sources: the pages "ssm_gdn_tc_route.rs" and "ssm_gdn_woa.rs"
 * (metrale_model_layers/layers/ops) and "ssm_ba_gates_hopper.rs"
 * (spark_model/layers/ops).
 */
#ifndef GDN_H_
#define GDN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* gdn_stream_t; /* same type as cudaStream_t */

/* Return codes. */
#define GDN_OK 0
#define GDN_ERR_NULL 1      /* a required pointer is NULL */
#define GDN_ERR_SHAPE 2     /* unsupported or inconsistent sizes */
#define GDN_ERR_STRIDE 3    /* a stride is shorter than its row */
#define GDN_ERR_WORKSPACE 4 /* workspace missing or too small */
#define GDN_ERR_CUDA 5      /* the CUDA runtime refused the launch */
#define GDN_ERR_ALIGN 6     /* pointer or stride breaks the 16-byte rule */

/* Bits of the verify/fold engaged word. */
#define GDN_FLAG_ENGAGED 1u /* a write-on-accept verify ran since the clear */
#define GDN_FLAG_ERROR 2u   /* a device-side guard fired (see each call) */
#define GDN_FLAG_STASH_BAD 4u /* a verify gave up (a bounded wait ran out) before its
                               * whole stash was written; always set together with
                               * GDN_FLAG_ERROR.  The fold then changes no state. */

/* Name of the guard that refused the last failing call on this thread, or ""
 * after a successful call.  Never NULL. */
const char* gdn_last_error(void);

/* Library version string ("gdn-b200 <major>.<minor>"). */
const char* gdn_version(void);

/* --------------------------------------------------------------------------
 * gdn_ba_gates -- the BA projection with its gate epilogue.
 * Page "ssm_ba_gates_hopper.rs": module doc (one BA output per (token, n),
 * n < N = 2*nv, each a dot product over the token's K-wide activation row),
 * the guards of ssm_ba_gates_hopper_reject, and ba_gates_slot (where output n
 * lands in the [gate(nv) | beta(nv)] row).
 *
 *   x        [M, k_stride] bf16; the reduction reads the first K of each row
 *   w_ba     [N, K] bf16 row-major (N = 2*nv)
 *   a_log    [nv] f32, dt_bias [nv] f32
 *   gate_out [M, gate_stride] f32: row m gets gate[0..nv) then beta[nv..2nv)
 *            with ba = x[m] . w_ba[n], within = n % (2*vpg), grp = n / (2*vpg):
 *              within <  vpg: beta[grp*vpg + within] = sigmoid(ba)
 *              within >= vpg: gate[grp*vpg + within - vpg]
 *                             = -exp(a_log[vh]) * softplus(ba + dt_bias[vh])
 * Errors: GDN_ERR_NULL (any pointer NULL), GDN_ERR_SHAPE (M < 0, N == 0,
 * K == 0, K % 8 != 0, N != 2*nv, vpg <= 0, nv % vpg != 0),
 * GDN_ERR_STRIDE (k_stride < K, gate_stride < 2*nv), GDN_ERR_ALIGN (x or w_ba
 * not 16-byte aligned, k_stride % 8 != 0).  M == 0 launches nothing.
 * ------------------------------------------------------------------------ */
int gdn_ba_gates(const uint16_t* x, int k_stride, const uint16_t* w_ba, const float* a_log,
                 const float* dt_bias, float* gate_out, int gate_stride, int M, int N, int K,
                 int nv, int vheads_per_group, gdn_stream_t stream);

/* --------------------------------------------------------------------------
 * gdn_chunk_prefill -- chunk-parallel varlen prefill (chunk C = 64).
 * Page "ssm_gdn_tc_route.rs": the prefill "state spine" chunk_delta_h carries
 * the f32 recurrent state across chunks; bf16 operands, f32 accumulation
 * ("f32 accumulator = the recurrent state, h stays f32").  Within a chunk the
 * WY/UT form is used; the result equals the token recurrence above up to
 * rounding.
 *
 *   q, k       [T, qk_stride] bf16; k-head hk of token t at t*qk_stride + hk*d_k
 *   v          [T, v_stride] bf16; v-head h at t*v_stride + h*d_v
 *   g, beta    [T, gb_stride] f32; head h at t*gb_stride + h.  Decay gates
 *              g <= 0 (the BA gates' range) are exact for any magnitude.
 *              Positive gates are exact while, within every 64-row chunk,
 *              the cumulative gate rises by at most 80 after any row
 *              (G_r - G_s <= 80 for s <= r, G_{-1} = 0); a larger rise
 *              overflows the f32 decay factors, so the kernel sets bit 64 of
 *              the prefill's device error word (gdn_debug_device_errors) and
 *              its results are undefined
 *   cu_seqlens [num_seqs + 1] int32 DEVICE array, cu[0] = 0, nondecreasing,
 *              cu[num_seqs] = total_tokens (empty sequences allowed)
 *   h0         [num_seqs, H_v, d_k, d_v] f32 initial states, or NULL = zeros
 *   hT         same shape, final states, or NULL = not stored; may equal h0
 *              (in-place update)
 *   o          [T, H_v, d_v] bf16 contiguous, round-to-nearest-even
 *   scale      multiplies every output (1.0 reproduces o_t = S_t q_t)
 *   workspace  device scratch of at least gdn_chunk_prefill_workspace_bytes()
 *              bytes, 256-byte aligned; its contents on entry do not matter
 * Supported: d_k == d_v in {64, 128}; H_v % H_k == 0; num_seqs >= 1.
 * Errors: GDN_ERR_NULL (q, k, v, g, beta, cu_seqlens or o NULL),
 * GDN_ERR_SHAPE, GDN_ERR_STRIDE (qk_stride < H_k*d_k, v_stride < H_v*d_v,
 * gb_stride < H_v), GDN_ERR_ALIGN (q/k/v/o/h0/hT not 16-byte aligned, or
 * qk_stride, v_stride not multiples of 8), GDN_ERR_WORKSPACE, GDN_ERR_CUDA.
 * total_tokens == 0 launches nothing except the copy h0 -> hT when both are
 * given and differ.
 * ------------------------------------------------------------------------ */
size_t gdn_chunk_prefill_workspace_bytes(int total_tokens, int num_seqs, int H_k, int H_v,
                                         int d_k, int d_v);
int gdn_chunk_prefill(const uint16_t* q, const uint16_t* k, int qk_stride, const uint16_t* v,
                      int v_stride, const float* g, const float* beta, int gb_stride,
                      const int32_t* cu_seqlens, int num_seqs, int total_tokens,
                      const float* h0, float* hT, uint16_t* o, int H_k, int H_v, int d_k,
                      int d_v, float scale, void* workspace, size_t workspace_bytes,
                      gdn_stream_t stream);

/* --------------------------------------------------------------------------
 * gdn_chunk_prefill_segmented -- the prefill as a segment-parallel
 * (two-level) scan with a given number of segments per sequence.
 * Page "ssm_gdn_tc_route.rs": the state spine carries the f32 state across
 * chunks, one chunk after the other.  Each chunk step is affine in the state
 * (H -> (e^{G_C} I - K~^T W) H + K~^T U), so a run of chunks is one affine map
 * H -> M H + L.  Each sequence is cut into `segments` runs of whole chunks;
 * the runs compute their L (from zero) and M (from the identity, with v
 * read as zeros) side by side, a short f32 combine gives every run its true
 * entry state, and the runs then produce their outputs from those states
 * side by side.  Chains are `segments` times shorter; the chunk work is
 * about three times the single-level scan's.  It pays when there are few
 * (sequence, v-head) units for the GPU -- e.g. a tensor-parallel shard that
 * holds a handful of heads -- and long sequences; gdn_chunk_prefill and
 * gdn_chunk_prefill_x2 take this path on their own exactly then.
 *
 *   segments   >= 1 (1 = the single-level scan of gdn_chunk_prefill); runs
 *              are ceil(chunks / segments) chunks long, the last ones may be
 *              shorter or empty
 *   limbs      1 (as gdn_chunk_prefill) or 2 (as gdn_chunk_prefill_x2)
 *   workspace  >= gdn_chunk_prefill_segmented_workspace_bytes(..., segments)
 *              bytes, 256-byte aligned (the runs' states live there)
 * Every other argument, guard and error is as for gdn_chunk_prefill;
 * GDN_ERR_SHAPE also for segments outside 1..64 or limbs outside 1..2.  The
 * result equals gdn_chunk_prefill's up to rounding (the combine adds one f32
 * product per run boundary).
 * ------------------------------------------------------------------------ */
size_t gdn_chunk_prefill_segmented_workspace_bytes(int total_tokens, int num_seqs, int H_k,
                                                   int H_v, int d_k, int d_v, int segments);
int gdn_chunk_prefill_segmented(const uint16_t* q, const uint16_t* k, int qk_stride,
                                const uint16_t* v, int v_stride, const float* g,
                                const float* beta, int gb_stride, const int32_t* cu_seqlens,
                                int num_seqs, int total_tokens, const float* h0, float* hT,
                                uint16_t* o, int H_k, int H_v, int d_k, int d_v, float scale,
                                int segments, int limbs, void* workspace,
                                size_t workspace_bytes, gdn_stream_t stream);

/* --------------------------------------------------------------------------
 * gdn_chunk_prefill_x2 -- gdn_chunk_prefill with a two-limb state operand.
 * Page "ssm_gdn_tc_route.rs": the tensor-core spine ships in two variants,
 * _tcfuse (one bf16 limb of S_c as the MMA operand) and _tcfuse_x2 (two bf16
 * limbs).  gdn_chunk_prefill is the one-limb spine; this entry point splits
 * the f32 state H into hi = bf16(H) and lo = bf16(H - hi) and feeds both to
 * the H-dependent products ([W; Q] H), so H enters them with ~16 bits of
 * mantissa instead of 8 (twice the MMA steps of that product).  The state
 * update itself is f32 in both.  Arguments, layouts, workspace, guards and
 * errors are exactly those of gdn_chunk_prefill.
 * ------------------------------------------------------------------------ */
int gdn_chunk_prefill_x2(const uint16_t* q, const uint16_t* k, int qk_stride, const uint16_t* v,
                         int v_stride, const float* g, const float* beta, int gb_stride,
                         const int32_t* cu_seqlens, int num_seqs, int total_tokens,
                         const float* h0, float* hT, uint16_t* o, int H_k, int H_v, int d_k,
                         int d_v, float scale, void* workspace, size_t workspace_bytes,
                         gdn_stream_t stream);

/* --------------------------------------------------------------------------
 * Write-on-accept speculative verify (K = 4 draft rows per sequence).
 * Page "ssm_gdn_woa.rs": gdn_decode_wy4_woa writes the outputs but no state,
 * stashes the per-row update terms for the fold, reaches each sequence's
 * state through a pointer table, and sets the engaged word.
 *
 * gdn_stash_seq_floats: floats of stash one sequence needs:
 *   H_v * 4 * (d_v + 4)  -- per head four delta rows then four cumulative
 *   gates, padded to a multiple of 4 floats.
 *
 *   h_table  [batch] device array of device pointers; entry b points at the
 *            state of sequence b, [H_v, d_k, d_v] f32, 16-byte aligned (the
 *            verify streams each state with bulk copies, the fold uses 16-byte
 *            accesses; entries live on the device, so this is not checked);
 *            a NULL entry marks a padding sequence (its o rows are written as
 *            zeros, nothing else)
 *   q, k     [batch*4, qk_stride] bf16; rows b*4 .. b*4+3 belong to sequence b
 *   v        [batch*4, v_stride] bf16; g, beta [batch*4, gb_stride] f32
 *   o        [batch*4, H_v, d_v] bf16
 *   stash    [batch * stash_seq_floats] f32 scratch owned by the caller,
 *            read by gdn_fold; stash_seq_floats >= gdn_stash_seq_floats(...)
 *   engaged_flag  u32: bit 0 is OR-ed in by every launched verify; a CTA
 *            whose bounded wait ran out ORs in GDN_FLAG_ERROR | GDN_FLAG_STASH_BAD
 * No state is written.  Supported: d_k == d_v in {64, 128}, H_v % H_k == 0.
 * Launch: min(batch * H_v, SM count) persistent CTAs of 512 threads walk the
 * (sequence, v-head) items; 211 KB (d = 128) of dynamic shared memory each.
 * Errors: GDN_ERR_NULL (h_table, stash, engaged_flag, q, k, v, g, beta or o
 * NULL -- the null guard of the page's launcher), GDN_ERR_SHAPE,
 * GDN_ERR_STRIDE, GDN_ERR_ALIGN, GDN_ERR_CUDA.  batch == 0 launches nothing.
 * ------------------------------------------------------------------------ */
int gdn_stash_seq_floats(int H_v, int d_k, int d_v);
int gdn_verify_woa(float* const* h_table, const uint16_t* q, const uint16_t* k, int qk_stride,
                   const uint16_t* v, int v_stride, const float* g, const float* beta,
                   int gb_stride, uint16_t* o, float* stash, int stash_seq_floats, int batch,
                   int H_k, int H_v, int d_k, int d_v, float scale, uint32_t* engaged_flag,
                   gdn_stream_t stream);

/* --------------------------------------------------------------------------
 * gdn_verify_woa_static -- gdn_verify_woa without a caller-provided stash.
 * No counterpart on the source pages: this entry point exists for callers
 * that cannot allocate device memory themselves -- for example an engine that
 * reserves all device memory up front in its own pool and forbids further
 * allocations while serving, or a latency-bound decode loop that must not
 * call cudaMalloc (which can synchronise the whole device).  Such a caller
 * still passes every input and output; only the stash (the scratch the verify
 * leaves for the fold) lives in the library.
 *
 * The stash is a static device array of GDN_STATIC_STASH_FLOATS f32 (8 MiB)
 * that every GPU loading this library holds until the process exits.
 * Sequence b uses floats [b * S, (b + 1) * S) with
 * S = gdn_stash_seq_floats(H_v, d_k, d_v); batch * S must not exceed
 * GDN_STATIC_STASH_FLOATS (GDN_ERR_SHAPE otherwise).  On success
 * *stash_out receives the array's device address: pass it, with
 * stash_seq_floats = S, to gdn_fold.  The first call on each device looks that
 * address up (cudaGetSymbolAddress, with the device current); make that first
 * call before any stream capture.  Nothing is allocated or freed, by this call
 * or by anything it calls.  All calls share the one array and it keeps the
 * last call's contents: a verify whose fold has not yet run must not be
 * followed by another static verify, and calls that overlap on the GPU (other
 * streams, other host threads) race on it.  Every other argument, guard and
 * error is as for gdn_verify_woa; stash_out must not be NULL.
 * ------------------------------------------------------------------------ */
#define GDN_STATIC_STASH_FLOATS (2u * 1024u * 1024u)
int gdn_verify_woa_static(float* const* h_table, const uint16_t* q, const uint16_t* k,
                          int qk_stride, const uint16_t* v, int v_stride, const float* g,
                          const float* beta, int gb_stride, uint16_t* o, int batch, int H_k,
                          int H_v, int d_k, int d_v, float scale, uint32_t* engaged_flag,
                          const float** stash_out, gdn_stream_t stream);

/* --------------------------------------------------------------------------
 * gdn_verify_parent -- the parent (not write-on-accept) K = 4 verify.
 * Page "ssm_gdn_woa.rs", gdn_wy4_fold doc: a clear engaged word means the
 * non-write-on-accept verify ran instead, and it left the intermediate states
 * Hi(i) in slabs reached through hi_tables, from which the fold restores a
 * partial accept.  This entry point is that verify: the same four rows as gdn_verify_woa (same outputs), but the
 * states are written instead of a stash:
 *     Hi(r) = state after rows 0..r  (r = 0..3, from H0 = the live state)
 *   - Hi(0), Hi(1), Hi(2) go to the slabs hi_tables[b * slab_entries + r]
 *     (a NULL entry, or hi_tables == NULL, keeps none of them),
 *   - Hi(3) replaces the live state h_table[b] in place.
 * It does not touch the engaged word: issue gdn_flag_clear before it, and the
 * fold's clear engaged bit then selects the restore branch.
 *
 *   h_table, q, k, v, g, beta, strides, o, batch, heads, scale: as for
 *            gdn_verify_woa (a NULL h_table entry is a padding sequence: zero
 *            outputs, no state written)
 *   hi_tables  [batch * slab_entries] device array of device pointers, entry
 *            b * slab_entries + r -> [H_v, d_k, d_v] f32, 16-byte aligned; or NULL
 *   slab_entries  entries per sequence, >= 3 when hi_tables is given
 * Traffic: each state is read once (plus an L2 re-read) and written up to four
 * times -- the cost the write-on-accept verify exists to avoid.
 * Errors: GDN_ERR_NULL (h_table, q, k, v, g, beta or o NULL), GDN_ERR_SHAPE,
 * GDN_ERR_STRIDE, GDN_ERR_CUDA.  batch == 0 launches nothing.
 * ------------------------------------------------------------------------ */
int gdn_verify_parent(float* const* h_table, const uint16_t* q, const uint16_t* k,
                      int qk_stride, const uint16_t* v, int v_stride, const float* g,
                      const float* beta, int gb_stride, uint16_t* o, float* const* hi_tables,
                      int slab_entries, int batch, int H_k, int H_v, int d_k, int d_v,
                      float scale, gdn_stream_t stream);

/* --------------------------------------------------------------------------
 * gdn_fold -- the post-verdict fold.
 * Page "ssm_gdn_woa.rs", gdn_wy4_fold, both branches, chosen on the device by
 * the engaged word:
 *  - engaged bit SET (a write-on-accept verify ran): apply the stashed rows
 *    0..na_tab[b] to H, reading and writing each touched state once:
 *        H <- exp(G_{na-1}) H + sum_{r<na} exp(G_{na-1} - G_r) k_r delta_r^T
 *    so H becomes the state after the first na rows.  na == 0 leaves H
 *    untouched (not even rewritten).  With GDN_FLAG_STASH_BAD set (the verify
 *    gave up part-way) no state is touched at all.
 *  - engaged bit CLEAR (the parent verify ran; the live state holds Hi(3)): a
 *    partial accept, 1 <= na < k_rows, copies Hi(na - 1) from
 *    hi_tables[b * slab_entries + na - 1] over the live state (bit for bit);
 *    na == k_rows leaves it as it is.  na == 0 cannot be restored (the state
 *    before the verify was overwritten) and, like a NULL slab entry, skips the
 *    sequence and sets GDN_FLAG_ERROR.  hi_tables == NULL makes this branch a
 *    no-op.
 * Either way H ends as the state after the first na rows.
 *
 *   h_table, stash, stash_seq_floats: as passed to gdn_verify_woa; stash and k
 *            may both be NULL when only the parent path is used (an engaged
 *            word then sets GDN_FLAG_ERROR and changes nothing)
 *   na_tab   [batch] int32 device array: accepted rows per sequence, 0..k_rows;
 *            a value outside 0..k_rows skips that sequence and sets
 *            GDN_FLAG_ERROR in the engaged word
 *   k        the same k rows the verify read (the stash holds delta and G only)
 *   hi_tables, slab_entries: as passed to gdn_verify_parent, or NULL / any
 *   engaged_flag  read; only GDN_FLAG_ERROR may be OR-ed in
 * Errors: GDN_ERR_NULL (h_table, na_tab or engaged_flag NULL; exactly one of
 * stash and k NULL; neither stash nor hi_tables given), GDN_ERR_SHAPE
 * (k_rows != 4, slab_entries < 3 with hi_tables, ...), GDN_ERR_STRIDE,
 * GDN_ERR_ALIGN, GDN_ERR_CUDA.
 * ------------------------------------------------------------------------ */
int gdn_fold(float* const* h_table, const float* stash, const int32_t* na_tab,
             const uint16_t* k, int qk_stride, float* const* hi_tables, int slab_entries,
             uint32_t* engaged_flag, int k_rows, int batch, int H_k, int H_v, int d_k, int d_v,
             int stash_seq_floats, gdn_stream_t stream);

/* --------------------------------------------------------------------------
 * gdn_flag_clear -- zero the engaged word on `stream`.
 * Page "ssm_gdn_woa.rs", gdn_wy4_flag_clear: issued at the start of a batched
 * verify, on the stream of the launches that follow.
 * Errors: GDN_ERR_NULL, GDN_ERR_CUDA.
 * ------------------------------------------------------------------------ */
int gdn_flag_clear(uint32_t* engaged_flag, gdn_stream_t stream);

/* --------------------------------------------------------------------------
 * gdn_debug_device_errors -- diagnostics, not part of the hot path.
 * Copies the library's four device-side error words (BA gates, prefill,
 * verify/fold, reserved) into host memory `out4` and clears them.  Bit 64 of
 * the prefill word means a gate rise beyond the documented bound (see
 * gdn_chunk_prefill); every other set bit means a bounded wait inside a kernel
 * gave up (the kernel then returned early instead of hanging).  This call
 * synchronises the device.
 * Errors: GDN_ERR_NULL, GDN_ERR_CUDA.
 * ------------------------------------------------------------------------ */
int gdn_debug_device_errors(uint32_t* out4);

/* --------------------------------------------------------------------------
 * gdn_debug_set_spin_limit -- diagnostics, not part of the hot path.
 * Every cross-CTA wait of the prefill's pipeline polls for at most a fixed
 * number of clock cycles (about 2 s) before it gives up: it then records a
 * bit in the prefill's device error word, raises the kernel's abort word and
 * every CTA returns -- the kernel never hangs.  This call sets that limit for
 * the prefill launches that follow (cycles > 0), or restores the default
 * (cycles == 0), so that a test can make the waits run out on purpose.  The
 * final drains of copies and MMAs still in flight always keep the default.
 * A process-wide setting, read at launch; not for concurrent use.
 * Errors: GDN_ERR_SHAPE (cycles < 0).
 * ------------------------------------------------------------------------ */
int gdn_debug_set_spin_limit(long long cycles);

#ifdef __cplusplus
}
#endif

#endif /* GDN_H_ */
