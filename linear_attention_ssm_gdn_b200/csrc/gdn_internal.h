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
                        const uint16_t* k, int qk_stride, uint32_t* flag, int k_rows,
                        int batch, int H_k, int H_v, int D, int stash_seq_floats,
                        cudaStream_t s);

size_t prefill_workspace_bytes(int total_tokens, int num_seqs, int H_k, int H_v, int D);

cudaError_t launch_prefill(const uint16_t* q, const uint16_t* k, int qk_stride,
                           const uint16_t* v, int v_stride, const float* g, const float* beta,
                           int gb_stride, const int32_t* cu_seqlens, int num_seqs,
                           int total_tokens, const float* h0, float* hT, uint16_t* o, int H_k,
                           int H_v, int D, float scale, void* workspace, cudaStream_t s);

// Device error words (one per kernel family): read and clear (synchronous).
cudaError_t take_err_ba_gates(uint32_t* out);
cudaError_t take_err_prefill(uint32_t* out);
cudaError_t take_err_verify(uint32_t* out);

}  // namespace gdn
