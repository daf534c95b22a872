// gdn_api.cu -- the extern "C" entry points of libgdn.so (declared in
// include/gdn.h): argument validation with named guards, then one launch on the
// caller's stream.  No entry point allocates, frees or synchronises (except the
// documented diagnostics call gdn_debug_device_errors).
//
// The guard style follows page "ssm_ba_gates_hopper.rs"
// (ssm_ba_gates_hopper_reject): every refusal names the guard that fired, so a
// rejected call can never pass silently as "no effect"; and page
// "ssm_gdn_woa.rs" (gdn_decode_wy4_woa's null table/stash/flag guard).
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <stdint.h>

#include <mutex>
#include <string>

#include "../../include/gdn.h"
#include "gdn_internal.h"

namespace gdn {

static thread_local std::string t_last_error;

void set_error(const std::string& msg) { t_last_error = msg; }
void clear_error() { t_last_error.clear(); }

static PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

bool encode_tmap_bf16(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                      const uint64_t* strides_bytes, const uint32_t* box, bool swizzle128) {
  auto fn = get_encode_fn();
  if (fn == nullptr) {
    set_error("cuTensorMapEncodeTiled unavailable from the driver");
    return false;
  }
  uint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, cuuint32_t(rank), const_cast<void*>(base),
                  reinterpret_cast<const cuuint64_t*>(dims),
                  reinterpret_cast<const cuuint64_t*>(strides_bytes),
                  reinterpret_cast<const cuuint32_t*>(box), estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    set_error("cuTensorMapEncodeTiled failed (code " + std::to_string(int(r)) + ")");
    return false;
  }
  return true;
}

int sm_count() {
  int dev = 0;
  cudaGetDevice(&dev);
  static int cache[64] = {0};
  if (dev < 0 || dev >= 64) return 148;
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

static cudaError_t read_device_errors(uint32_t* out4) {
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return e;
  out4[3] = 0;
  if ((e = take_err_ba_gates(&out4[0])) != cudaSuccess) return e;
  if ((e = take_err_prefill(&out4[1])) != cudaSuccess) return e;
  return take_err_verify(&out4[2]);
}

}  // namespace gdn

using gdn::set_error;

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int fail(int code, const std::string& msg) {
  set_error(msg);
  return code;
}

int cuda_status(cudaError_t e, const char* what) {
  if (e != cudaSuccess)
    return fail(GDN_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
  gdn::clear_error();
  return GDN_OK;
}

// Head geometry shared by prefill / verify / fold.
int check_heads(const char* fn, int H_k, int H_v, int d_k, int d_v) {
  if (H_k <= 0 || H_v <= 0) return fail(GDN_ERR_SHAPE, std::string(fn) + ": H_k and H_v must be > 0");
  if (H_v % H_k != 0)
    return fail(GDN_ERR_SHAPE, std::string(fn) + ": H_v is not a multiple of H_k");
  if (d_k != d_v || (d_k != 64 && d_k != 128))
    return fail(GDN_ERR_SHAPE, std::string(fn) + ": need d_k == d_v in {64, 128}");
  return GDN_OK;
}

}  // namespace

extern "C" {

const char* gdn_last_error(void) { return gdn::t_last_error.c_str(); }

const char* gdn_version(void) { return "gdn-b200 0.1"; }

int gdn_ba_gates(const uint16_t* x, int k_stride, const uint16_t* w_ba, const float* a_log,
                 const float* dt_bias, float* gate_out, int gate_stride, int M, int N, int K,
                 int nv, int vheads_per_group, gdn_stream_t stream) {
  if (!x || !w_ba || !a_log || !dt_bias || !gate_out)
    return fail(GDN_ERR_NULL, "gdn_ba_gates: null x/w_ba/a_log/dt_bias/gate_out");
  if (M < 0) return fail(GDN_ERR_SHAPE, "gdn_ba_gates: M < 0");
  if (N == 0 || K == 0) return fail(GDN_ERR_SHAPE, "gdn_ba_gates: empty BA projection");
  if (N < 0 || K < 0) return fail(GDN_ERR_SHAPE, "gdn_ba_gates: negative N or K");
  if (K % 8 != 0)
    return fail(GDN_ERR_SHAPE, "gdn_ba_gates: K is not a multiple of 8 (16-byte row tiles)");
  if (N != 2 * nv) return fail(GDN_ERR_SHAPE, "gdn_ba_gates: N != 2*nv");
  if (N > 256) return fail(GDN_ERR_SHAPE, "gdn_ba_gates: N > 256 (one MMA tile)");
  if (vheads_per_group <= 0 || nv % vheads_per_group != 0)
    return fail(GDN_ERR_SHAPE, "gdn_ba_gates: nv is not a multiple of vheads_per_group");
  if (k_stride < K)
    return fail(GDN_ERR_STRIDE,
                "gdn_ba_gates: K_stride < K: the activation row is shorter than the reduction");
  if (gate_stride < 2 * nv) return fail(GDN_ERR_STRIDE, "gdn_ba_gates: gate_stride < 2*nv");
  if (!aligned16(x) || !aligned16(w_ba) || k_stride % 8 != 0)
    return fail(GDN_ERR_ALIGN, "gdn_ba_gates: x/w_ba not 16-byte aligned or k_stride % 8 != 0");
  if (M == 0) {
    gdn::clear_error();
    return GDN_OK;
  }
  return cuda_status(gdn::launch_ba_gates(x, k_stride, w_ba, a_log, dt_bias, gate_out,
                                          gate_stride, M, N, K, nv, vheads_per_group,
                                          reinterpret_cast<cudaStream_t>(stream)),
                     "gdn_ba_gates");
}

// Workspace of a prefill call with `segments` segments per sequence
// (1: single level; the segmented path also needs the per-segment states).
static size_t prefill_need(int total_tokens, int num_seqs, int H_v, int d_k, int segments) {
  if (segments <= 1) return gdn::prefill_ring_bytes(num_seqs * H_v);
  return gdn::prefill_segmented_workspace_bytes(total_tokens, num_seqs, H_v, d_k, segments);
}

static int auto_segments(int total_tokens, int num_seqs, int H_v) {
  if (num_seqs <= 0 || H_v <= 0 || total_tokens <= 0) return 1;
  return gdn::prefill_auto_segments(total_tokens, num_seqs, H_v);
}

size_t gdn_chunk_prefill_workspace_bytes(int total_tokens, int num_seqs, int H_k, int H_v,
                                         int d_k, int d_v) {
  (void)H_k;
  (void)d_v;
  if (num_seqs <= 0 || H_v <= 0) return 0;
  return prefill_need(total_tokens, num_seqs, H_v, d_k,
                      auto_segments(total_tokens, num_seqs, H_v));
}

size_t gdn_chunk_prefill_segmented_workspace_bytes(int total_tokens, int num_seqs, int H_k,
                                                   int H_v, int d_k, int d_v, int segments) {
  (void)H_k;
  (void)d_v;
  if (num_seqs <= 0 || H_v <= 0 || segments < 1) return 0;
  return prefill_need(total_tokens, num_seqs, H_v, d_k, segments);
}

// segments: >= 1 as given, 0 = the library's choice.
static int chunk_prefill(const char* fn, int limbs, int segments, const uint16_t* q,
                         const uint16_t* k, int qk_stride, const uint16_t* v, int v_stride,
                         const float* g, const float* beta, int gb_stride,
                         const int32_t* cu_seqlens, int num_seqs, int total_tokens,
                         const float* h0, float* hT, uint16_t* o, int H_k, int H_v, int d_k,
                         int d_v, float scale, void* workspace, size_t workspace_bytes,
                         gdn_stream_t stream) {
  const std::string f(fn);
  if (!q || !k || !v || !g || !beta || !cu_seqlens || !o)
    return fail(GDN_ERR_NULL, f + ": null q/k/v/g/beta/cu_seqlens/o");
  int rc = check_heads(fn, H_k, H_v, d_k, d_v);
  if (rc != GDN_OK) return rc;
  if (num_seqs <= 0) return fail(GDN_ERR_SHAPE, f + ": num_seqs must be >= 1");
  if (total_tokens < 0) return fail(GDN_ERR_SHAPE, f + ": total_tokens < 0");
  if (segments < 0 || segments > 64)
    return fail(GDN_ERR_SHAPE, f + ": segments must be in 0..64");
  if (qk_stride < H_k * d_k) return fail(GDN_ERR_STRIDE, f + ": qk_stride < H_k*d_k");
  if (v_stride < H_v * d_v) return fail(GDN_ERR_STRIDE, f + ": v_stride < H_v*d_v");
  if (gb_stride < H_v) return fail(GDN_ERR_STRIDE, f + ": gb_stride < H_v");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) ||
      (h0 && !aligned16(h0)) || (hT && !aligned16(hT)))
    return fail(GDN_ERR_ALIGN, f + ": q/k/v/o/h0/hT not 16-byte aligned");
  if (qk_stride % 8 != 0 || v_stride % 8 != 0)
    return fail(GDN_ERR_ALIGN, f + ": qk_stride and v_stride must be multiples of 8");
  const int S = segments == 0 ? auto_segments(total_tokens, num_seqs, H_v) : segments;
  const size_t need = prefill_need(total_tokens, num_seqs, H_v, d_k, S);
  if (need > 0 && (workspace == nullptr || workspace_bytes < need ||
                   (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0))
    return fail(GDN_ERR_WORKSPACE, f + ": workspace missing, small or unaligned");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (total_tokens == 0) {
    if (hT != nullptr && hT != h0) {
      const size_t bytes = size_t(num_seqs) * H_v * d_k * d_v * sizeof(float);
      cudaError_t e = h0 ? cudaMemcpyAsync(hT, h0, bytes, cudaMemcpyDeviceToDevice, s)
                         : cudaMemsetAsync(hT, 0, bytes, s);
      return cuda_status(e, fn);
    }
    gdn::clear_error();
    return GDN_OK;
  }
  gdn::PrefillCall c = {};
  c.q = q;
  c.k = k;
  c.v = v;
  c.qk_stride = qk_stride;
  c.v_stride = v_stride;
  c.g = g;
  c.beta = beta;
  c.gb_stride = gb_stride;
  c.cu_seqlens = cu_seqlens;
  c.num_seqs = num_seqs;
  c.total_tokens = total_tokens;
  c.h0 = h0;
  c.hT = hT;
  c.o = o;
  c.H_k = H_k;
  c.H_v = H_v;
  c.D = d_k;
  c.scale = scale;
  c.limbs = limbs;
  c.workspace = workspace;
  if (S >= 2) return cuda_status(gdn::launch_prefill_segmented(c, S, workspace, s), fn);
  return cuda_status(gdn::launch_prefill_call(c, s), fn);
}

int gdn_chunk_prefill(const uint16_t* q, const uint16_t* k, int qk_stride, const uint16_t* v,
                      int v_stride, const float* g, const float* beta, int gb_stride,
                      const int32_t* cu_seqlens, int num_seqs, int total_tokens,
                      const float* h0, float* hT, uint16_t* o, int H_k, int H_v, int d_k,
                      int d_v, float scale, void* workspace, size_t workspace_bytes,
                      gdn_stream_t stream) {
  return chunk_prefill("gdn_chunk_prefill", 1, 0, q, k, qk_stride, v, v_stride, g, beta,
                       gb_stride, cu_seqlens, num_seqs, total_tokens, h0, hT, o, H_k, H_v, d_k,
                       d_v, scale, workspace, workspace_bytes, stream);
}

int gdn_chunk_prefill_x2(const uint16_t* q, const uint16_t* k, int qk_stride, const uint16_t* v,
                         int v_stride, const float* g, const float* beta, int gb_stride,
                         const int32_t* cu_seqlens, int num_seqs, int total_tokens,
                         const float* h0, float* hT, uint16_t* o, int H_k, int H_v, int d_k,
                         int d_v, float scale, void* workspace, size_t workspace_bytes,
                         gdn_stream_t stream) {
  return chunk_prefill("gdn_chunk_prefill_x2", 2, 0, q, k, qk_stride, v, v_stride, g, beta,
                       gb_stride, cu_seqlens, num_seqs, total_tokens, h0, hT, o, H_k, H_v, d_k,
                       d_v, scale, workspace, workspace_bytes, stream);
}

int gdn_chunk_prefill_segmented(const uint16_t* q, const uint16_t* k, int qk_stride,
                                const uint16_t* v, int v_stride, const float* g,
                                const float* beta, int gb_stride, const int32_t* cu_seqlens,
                                int num_seqs, int total_tokens, const float* h0, float* hT,
                                uint16_t* o, int H_k, int H_v, int d_k, int d_v, float scale,
                                int segments, int limbs, void* workspace,
                                size_t workspace_bytes, gdn_stream_t stream) {
  if (segments < 1)
    return fail(GDN_ERR_SHAPE, "gdn_chunk_prefill_segmented: segments must be >= 1");
  if (limbs != 1 && limbs != 2)
    return fail(GDN_ERR_SHAPE, "gdn_chunk_prefill_segmented: limbs must be 1 or 2");
  return chunk_prefill("gdn_chunk_prefill_segmented", limbs, segments, q, k, qk_stride, v,
                       v_stride, g, beta, gb_stride, cu_seqlens, num_seqs, total_tokens, h0, hT,
                       o, H_k, H_v, d_k, d_v, scale, workspace, workspace_bytes, stream);
}

int gdn_stash_seq_floats(int H_v, int d_k, int d_v) {
  (void)d_k;
  return H_v * 4 * (d_v + 4);
}

int gdn_verify_woa(float* const* h_table, const uint16_t* q, const uint16_t* k, int qk_stride,
                   const uint16_t* v, int v_stride, const float* g, const float* beta,
                   int gb_stride, uint16_t* o, float* stash, int stash_seq_floats, int batch,
                   int H_k, int H_v, int d_k, int d_v, float scale, uint32_t* engaged_flag,
                   gdn_stream_t stream) {
  const char* fn = "gdn_verify_woa";
  if (!h_table || !stash || !engaged_flag)
    return fail(GDN_ERR_NULL, "gdn_verify_woa: null table/stash/flag");
  if (!q || !k || !v || !g || !beta || !o)
    return fail(GDN_ERR_NULL, "gdn_verify_woa: null q/k/v/g/beta/o");
  int rc = check_heads(fn, H_k, H_v, d_k, d_v);
  if (rc != GDN_OK) return rc;
  if (batch < 0) return fail(GDN_ERR_SHAPE, "gdn_verify_woa: batch < 0");
  if (qk_stride < H_k * d_k || v_stride < H_v * d_v || gb_stride < H_v)
    return fail(GDN_ERR_STRIDE, "gdn_verify_woa: a stride is shorter than its row");
  if (stash_seq_floats < gdn_stash_seq_floats(H_v, d_k, d_v))
    return fail(GDN_ERR_SHAPE, "gdn_verify_woa: stash_seq_floats < gdn_stash_seq_floats()");
  if (!aligned16(stash)) return fail(GDN_ERR_ALIGN, "gdn_verify_woa: stash not 16-byte aligned");
  if (batch == 0) {
    gdn::clear_error();
    return GDN_OK;
  }
  return cuda_status(gdn::launch_verify(h_table, q, k, qk_stride, v, v_stride, g, beta, gb_stride,
                                        o, stash, stash_seq_floats, batch, H_k, H_v, d_k, scale,
                                        engaged_flag, reinterpret_cast<cudaStream_t>(stream)),
                     fn);
}

int gdn_verify_woa_static(float* const* h_table, const uint16_t* q, const uint16_t* k,
                          int qk_stride, const uint16_t* v, int v_stride, const float* g,
                          const float* beta, int gb_stride, uint16_t* o, int batch, int H_k,
                          int H_v, int d_k, int d_v, float scale, uint32_t* engaged_flag,
                          const float** stash_out, gdn_stream_t stream) {
  const char* fn = "gdn_verify_woa_static";
  if (!stash_out) return fail(GDN_ERR_NULL, "gdn_verify_woa_static: null stash_out");
  if (!h_table || !engaged_flag)
    return fail(GDN_ERR_NULL, "gdn_verify_woa_static: null table/flag");
  if (!q || !k || !v || !g || !beta || !o)
    return fail(GDN_ERR_NULL, "gdn_verify_woa_static: null q/k/v/g/beta/o");
  int rc = check_heads(fn, H_k, H_v, d_k, d_v);
  if (rc != GDN_OK) return rc;
  if (batch < 0) return fail(GDN_ERR_SHAPE, "gdn_verify_woa_static: batch < 0");
  if (qk_stride < H_k * d_k || v_stride < H_v * d_v || gb_stride < H_v)
    return fail(GDN_ERR_STRIDE, "gdn_verify_woa_static: a stride is shorter than its row");
  const int ssf = gdn_stash_seq_floats(H_v, d_k, d_v);
  if (size_t(batch) * size_t(ssf) > gdn::static_stash_floats())
    return fail(GDN_ERR_SHAPE,
                "gdn_verify_woa_static: batch * gdn_stash_seq_floats() exceeds the static stash "
                "(GDN_STATIC_STASH_FLOATS = 2 Mi floats, 8 MiB)");
  float* stash = nullptr;
  cudaError_t e = gdn::static_stash_address(&stash);
  if (e != cudaSuccess) return cuda_status(e, fn);
  *stash_out = stash;
  if (batch == 0) {
    gdn::clear_error();
    return GDN_OK;
  }
  return cuda_status(gdn::launch_verify(h_table, q, k, qk_stride, v, v_stride, g, beta, gb_stride,
                                        o, stash, ssf, batch, H_k, H_v, d_k, scale, engaged_flag,
                                        reinterpret_cast<cudaStream_t>(stream)),
                     fn);
}

int gdn_verify_parent(float* const* h_table, const uint16_t* q, const uint16_t* k,
                      int qk_stride, const uint16_t* v, int v_stride, const float* g,
                      const float* beta, int gb_stride, uint16_t* o, float* const* hi_tables,
                      int slab_entries, int batch, int H_k, int H_v, int d_k, int d_v,
                      float scale, gdn_stream_t stream) {
  const char* fn = "gdn_verify_parent";
  if (!h_table) return fail(GDN_ERR_NULL, "gdn_verify_parent: null table");
  if (!q || !k || !v || !g || !beta || !o)
    return fail(GDN_ERR_NULL, "gdn_verify_parent: null q/k/v/g/beta/o");
  int rc = check_heads(fn, H_k, H_v, d_k, d_v);
  if (rc != GDN_OK) return rc;
  if (batch < 0) return fail(GDN_ERR_SHAPE, "gdn_verify_parent: batch < 0");
  if (hi_tables != nullptr && slab_entries < 3)
    return fail(GDN_ERR_SHAPE, "gdn_verify_parent: slab_entries < k_rows - 1 = 3");
  if (qk_stride < H_k * d_k || v_stride < H_v * d_v || gb_stride < H_v)
    return fail(GDN_ERR_STRIDE, "gdn_verify_parent: a stride is shorter than its row");
  if (batch == 0) {
    gdn::clear_error();
    return GDN_OK;
  }
  return cuda_status(gdn::launch_verify_parent(h_table, q, k, qk_stride, v, v_stride, g, beta,
                                               gb_stride, o, hi_tables, slab_entries, batch, H_k,
                                               H_v, d_k, scale,
                                               reinterpret_cast<cudaStream_t>(stream)),
                     fn);
}

int gdn_fold(float* const* h_table, const float* stash, const int32_t* na_tab,
             const uint16_t* k, int qk_stride, float* const* hi_tables, int slab_entries,
             uint32_t* engaged_flag, int k_rows, int batch, int H_k, int H_v, int d_k, int d_v,
             int stash_seq_floats, gdn_stream_t stream) {
  const char* fn = "gdn_fold";
  if (!h_table || !na_tab || !engaged_flag)
    return fail(GDN_ERR_NULL, "gdn_fold: null table/na_tab/flag");
  if ((stash == nullptr) != (k == nullptr))
    return fail(GDN_ERR_NULL, "gdn_fold: stash and k must both be given or both be NULL");
  if (stash == nullptr && hi_tables == nullptr)
    return fail(GDN_ERR_NULL, "gdn_fold: neither a stash (write-on-accept) nor hi_tables (parent)");
  int rc = check_heads(fn, H_k, H_v, d_k, d_v);
  if (rc != GDN_OK) return rc;
  if (k_rows != 4) return fail(GDN_ERR_SHAPE, "gdn_fold: k_rows must be 4");
  if (batch < 0) return fail(GDN_ERR_SHAPE, "gdn_fold: batch < 0");
  if (hi_tables != nullptr && slab_entries < k_rows - 1)
    return fail(GDN_ERR_SHAPE, "gdn_fold: slab_entries < k_rows - 1");
  if (stash != nullptr) {
    if (qk_stride < H_k * d_k) return fail(GDN_ERR_STRIDE, "gdn_fold: qk_stride < H_k*d_k");
    if (stash_seq_floats < gdn_stash_seq_floats(H_v, d_k, d_v))
      return fail(GDN_ERR_SHAPE, "gdn_fold: stash_seq_floats < gdn_stash_seq_floats()");
    if (!aligned16(stash)) return fail(GDN_ERR_ALIGN, "gdn_fold: stash not 16-byte aligned");
  }
  if (batch == 0) {
    gdn::clear_error();
    return GDN_OK;
  }
  return cuda_status(gdn::launch_fold(h_table, stash, na_tab, k, qk_stride, hi_tables,
                                      slab_entries, engaged_flag, k_rows, batch, H_k, H_v, d_k,
                                      stash_seq_floats, reinterpret_cast<cudaStream_t>(stream)),
                     fn);
}

int gdn_flag_clear(uint32_t* engaged_flag, gdn_stream_t stream) {
  if (!engaged_flag) return fail(GDN_ERR_NULL, "gdn_flag_clear: null flag");
  return cuda_status(gdn::launch_flag_clear(engaged_flag, reinterpret_cast<cudaStream_t>(stream)),
                     "gdn_flag_clear");
}

int gdn_debug_set_spin_limit(long long cycles) {
  if (cycles < 0) return fail(GDN_ERR_SHAPE, "gdn_debug_set_spin_limit: cycles < 0");
  gdn::set_prefill_spin_limit(cycles);
  gdn::clear_error();
  return GDN_OK;
}

int gdn_debug_device_errors(uint32_t* out4) {
  if (!out4) return fail(GDN_ERR_NULL, "gdn_debug_device_errors: null out4");
  return cuda_status(gdn::read_device_errors(out4), "gdn_debug_device_errors");
}

}  // extern "C"
