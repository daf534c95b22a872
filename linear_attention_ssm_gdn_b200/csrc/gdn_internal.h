// gdn_internal.h -- host-side glue shared by the translation units of
// libgdn.so (launchers, tensor-map encoding, error reporting).  Not part of
// the public ABI; the public declarations are in include/gdn.h.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <string>

namespace gdn {

// Thread-local "last error" text behind gdn_last_error().
void set_error(const std::string& msg);
void clear_error();

// Encode a bf16 tensor map with 128-byte swizzle.  dims/strides follow the
// driver's convention: dims[0] is innermost; strides_bytes[i] is the stride of
// dimension i+1.  Returns false (and sets the error text) on failure.
bool encode_tmap_bf16(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                      const uint64_t* strides_bytes, const uint32_t* box, bool swizzle128);

// Number of SMs of the current device (cached per device).
int sm_count();

// Launchers (validate nothing; gdn_api.cu has already checked every argument).
cudaError_t launch_ba_gates(const uint16_t* x, int k_stride, const uint16_t* w,
                            const float* a_log, const float* dt_bias, float* out,
                            int gate_stride, int M, int N, int K, int nv, int vpg,
                            cudaStream_t s);

cudaError_t launch_flag_clear(uint32_t* flag, cudaStream_t s);

cudaError_t launch_verify(float* const* h_table, const uint16_t* q, const uint16_t* k,
                          int qk_stride, const uint16_t* v, int v_stride, const float* g,
                          const float* beta, int gb_stride, uint16_t* o, float* stash,
                          int stash_seq_floats, int batch, int H_k, int H_v, int D, float scale,
                          uint32_t* flag, cudaStream_t s);

// Device address of the library-owned verify stash on the current device
// (looked up once per device); nullptr and the error on failure.
cudaError_t static_stash_address(float** out);
size_t static_stash_floats();

cudaError_t launch_fold(float* const* h_table, const float* stash, const int32_t* na_tab,
                        const uint16_t* k, int qk_stride, float* const* hi_tables,
                        int slab_entries, uint32_t* flag, int k_rows, int batch, int H_k,
                        int H_v, int D, int stash_seq_floats, cudaStream_t s);

cudaError_t launch_verify_parent(float* const* h_table, const uint16_t* q, const uint16_t* k,
                                 int qk_stride, const uint16_t* v, int v_stride, const float* g,
                                 const float* beta, int gb_stride, uint16_t* o,
                                 float* const* hi_tables, int slab_entries, int batch, int H_k,
                                 int H_v, int D, float scale, cudaStream_t s);

// One launch of the chunk-parallel prefill kernel.  The optional per-sequence
// overrides (seg, h0_tab, hT_tab, v_zero) let the segment-parallel scan run it
// over segments of the caller's sequences; plain calls leave them NULL / 0.
struct PrefillCall {
  const uint16_t* q;
  const uint16_t* k;
  const uint16_t* v;
  int qk_stride, v_stride;
  const float* g;
  const float* beta;
  int gb_stride;
  const int32_t* cu_seqlens;  // [num_seqs + 1], unless seg is given
  const int2* seg;            // [num_seqs] token ranges [x, y), or NULL
  int num_seqs, total_tokens;
  const float* h0;            // [num_seqs, H_v, D, D] or NULL (zeros)
  float* hT;                  // same, or NULL (not stored)
  const float* const* h0_tab; // [num_seqs] per-sequence overrides of h0 (NULL entry = zeros)
  float* const* hT_tab;       // [num_seqs] per-sequence overrides of hT (NULL entry = not stored)
  uint16_t* o;                // [total_tokens, H_v, D], or NULL (not stored)
  int v_zero;                 // 1: v is read as zeros
  int h0_identity;            // 1: every initial state is the identity (d_k == d_v)
  int H_k, H_v, D;
  float scale;
  int limbs;                  // 1 or 2 bf16 limbs of the state in the MMAs
  void* workspace;            // >= prefill_ring_bytes(num_seqs * H_v), 256-byte aligned
};

// Workspace (hand-off flags + L2 ring) of one launch over `units` (sequence,
// v-head) units; the most spines a launch uses.
size_t prefill_ring_bytes(int units);
void set_prefill_spin_limit(long long cycles);  // 0: the default (about 2 s)
int prefill_spine_budget();
cudaError_t launch_prefill_call(const PrefillCall& c, cudaStream_t s);

// The segment-parallel (two-level) scan over `segments` >= 2 segments per
// sequence (gdn_segmented.cu); workspace query and launch.
size_t prefill_segmented_workspace_bytes(int total_tokens, int num_seqs, int H_v, int D,
                                         int segments);
cudaError_t launch_prefill_segmented(const PrefillCall& c, int segments, void* workspace,
                                     cudaStream_t s);
// Segments the library picks on its own for a call (1: the single-level path).
int prefill_auto_segments(int total_tokens, int num_seqs, int H_v);

// Device error words (one per kernel family): read and clear (synchronous).
cudaError_t take_err_ba_gates(uint32_t* out);
cudaError_t take_err_prefill(uint32_t* out);
cudaError_t take_err_verify(uint32_t* out);

}  // namespace gdn
