// gdn_verify.cu -- K=4 write-on-accept verify, the post-verdict fold and the
// engaged-word clear (page "ssm_gdn_woa.rs": gdn_decode_wy4_woa, gdn_wy4_fold,
// gdn_wy4_flag_clear).
//
// Verify.  For sequence b (rows b*4+r, r < 4) and v-head h, with H0 = the state
// behind h_table[b] (f32 [d_k][d_v], H = S^T), G_r = g_0 + ... + g_r, and the
// scalars kk[s][r] = k_s.k_r, kq[s][r] = k_s.q_r, every state column j runs
// its own 4-step recurrence:
//   a_r[j] = (S0 k_r)_j = sum_i H0[i][j] k_r[i],   b_r[j] = (S0 q_r)_j
//   delta_r[j] = beta_r (v_r[j] - e^{G_r} a_r[j]
//                          - sum_{s<r} e^{G_r - G_s} kk[s][r] delta_s[j])
//   o_r[j] = scale (e^{G_r} b_r[j] + sum_{s<=r} e^{G_r - G_s} kq[s][r] delta_s[j])
// which is the token recurrence unrolled over four rows.  H0 is read once
// (16-byte loads, 4 columns per thread, 8 row groups per CTA, every load of a
// thread in flight at once); nothing is written to it.  delta_r and G_r go to
// the stash for the fold.
//
// Fold.  With na = na_tab[b] in 1..4 (and the engaged bit set):
//   H[i][j] <- e^{G_{na-1}} H[i][j] + sum_{r<na} e^{G_{na-1} - G_r} k_r[i] delta_r[j]
// reading and writing each state element once; na = 0 touches nothing.
// All of this is HBM-bound CUDA-core work: 4 rows give 8 flops per state
// element, far below the tensor-core ridge.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <mutex>

#include "gdn_device.cuh"
#include "gdn_internal.h"

namespace gdn {

__device__ uint32_t g_err_verify;

// The verify stash for callers that cannot allocate (gdn_verify_woa_static):
// 2 Mi floats = 8 MiB, held by every device that loads the library.
constexpr size_t kStaticStashFloats = size_t(2) * 1024 * 1024;
static __device__ __align__(256) float g_static_stash[kStaticStashFloats];

constexpr uint32_t kFlagEngaged = 1u;
constexpr uint32_t kFlagError = 2u;
constexpr int kRows = 4;

__device__ __forceinline__ float bf16_at(const uint16_t* p) {
  return __uint_as_float(uint32_t(*p) << 16);
}

__global__ void flag_clear_kernel(uint32_t* flag) {
  if (threadIdx.x == 0) *flag = 0u;
}

constexpr int kVThreads = 256;

// grid = (H_v, batch); block = 256 threads = GROUPS row groups x QUADS column
// quads.  Every thread issues all of its state loads (16 x 16 bytes at
// d = 128) before it needs any of them, so a CTA waits for memory about once;
// four CTAs per SM (64 registers) keep the loads of one CTA overlapping the
// recurrence of another (measured: 55.6 us against 75.4 us at two per SM).
template <int D>
__global__ void __launch_bounds__(kVThreads, 4) verify_kernel(
    float* const* __restrict__ h_table, const uint16_t* __restrict__ q,
    const uint16_t* __restrict__ k, int qk_stride, const uint16_t* __restrict__ v, int v_stride,
    const float* __restrict__ g, const float* __restrict__ beta, int gb_stride,
    uint16_t* __restrict__ o, float* __restrict__ stash, int stash_seq_floats, int H_k, int H_v,
    float scale, uint32_t* flag) {
  constexpr int QUADS = D / 4;              // column quads per row
  constexpr int GROUPS = kVThreads / QUADS;  // row groups (8 for D=128, 16 for D=64)
  constexpr int RPG = D / GROUPS;            // rows per group (16 resp. 4)
  __shared__ float ks[kRows][D], qs[kRows][D];
  __shared__ float4 part[GROUPS][2 * kRows][QUADS];  // partial a_r, b_r per row group
  __shared__ float kk[kRows][kRows], kq[kRows][kRows], G[kRows], bt[kRows];

  const int h = blockIdx.x, b = blockIdx.y;
  const int hk = h / (H_v / H_k);
  const int tid = threadIdx.x;
  const int quad = tid % QUADS, grp = tid / QUADS;
  const float* H0 = h_table[b];
  if (b == 0 && h == 0 && tid == 0) atomicOr(flag, kFlagEngaged);

  const size_t row0 = size_t(b) * kRows;
  if (H0 == nullptr) {  // padding sequence: zero outputs, nothing else
    for (int idx = tid; idx < kRows * D; idx += kVThreads) {
      const int r = idx / D, j = idx % D;
      o[((row0 + r) * H_v + h) * D + j] = 0;
    }
    return;
  }
  // This thread's rows of the state, all loads in flight at once.
  const float4* H4 = reinterpret_cast<const float4*>(H0 + size_t(h) * D * D);
  float4 hv[RPG];
#pragma unroll
  for (int ii = 0; ii < RPG; ++ii) hv[ii] = __ldg(&H4[(grp * RPG + ii) * QUADS + quad]);
  // v for the recurrence (thread j < D owns column j)
  float vr[kRows];
#pragma unroll
  for (int r = 0; r < kRows; ++r)
    vr[r] = tid < D ? bf16_at(v + (row0 + r) * v_stride + size_t(h) * D + tid) : 0.f;
  for (int idx = tid; idx < kRows * D; idx += kVThreads) {
    const int r = idx / D, i = idx % D;
    ks[r][i] = bf16_at(k + (row0 + r) * qk_stride + size_t(hk) * D + i);
    qs[r][i] = bf16_at(q + (row0 + r) * qk_stride + size_t(hk) * D + i);
  }
  if (tid < kRows) {
    G[tid] = g[(row0 + tid) * gb_stride + h];
    bt[tid] = beta[(row0 + tid) * gb_stride + h];
  }
  __syncthreads();
  if (tid == 0) {
    float run = 0.f;
    for (int r = 0; r < kRows; ++r) {
      run += G[r];
      G[r] = run;
    }
  }
  if (tid >= 64 && tid < 64 + 2 * kRows * kRows) {  // 16 k.k and 16 k.q dot products
    const int t = tid - 64;
    const int which = t / (kRows * kRows), s = (t / kRows) % kRows, r = t % kRows;
    float acc = 0.f;
    const float* other = which == 0 ? ks[r] : qs[r];
    for (int i = 0; i < D; ++i) acc = fmaf(ks[s][i], other[i], acc);
    if (which == 0)
      kk[s][r] = acc;
    else
      kq[s][r] = acc;
  }
  // a_r, b_r partial sums over this thread's rows for its 4 columns.
  float4 acc[2 * kRows];
#pragma unroll
  for (int r = 0; r < 2 * kRows; ++r) acc[r] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int ii = 0; ii < RPG; ++ii) {
    const int i = grp * RPG + ii;
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
      const float kv = ks[r][i], qv = qs[r][i];
      acc[r].x = fmaf(hv[ii].x, kv, acc[r].x);
      acc[r].y = fmaf(hv[ii].y, kv, acc[r].y);
      acc[r].z = fmaf(hv[ii].z, kv, acc[r].z);
      acc[r].w = fmaf(hv[ii].w, kv, acc[r].w);
      acc[kRows + r].x = fmaf(hv[ii].x, qv, acc[kRows + r].x);
      acc[kRows + r].y = fmaf(hv[ii].y, qv, acc[kRows + r].y);
      acc[kRows + r].z = fmaf(hv[ii].z, qv, acc[kRows + r].z);
      acc[kRows + r].w = fmaf(hv[ii].w, qv, acc[kRows + r].w);
    }
  }
#pragma unroll
  for (int r = 0; r < 2 * kRows; ++r) part[grp][r][quad] = acc[r];
  __syncthreads();
  // One thread per column: reduce the row groups, run the 4-step recurrence.
  if (tid < D) {
    const int j = tid;
    float a[kRows], bq[kRows], delta[kRows];
#pragma unroll
    for (int r = 0; r < 2 * kRows; ++r) {
      float s = 0.f;
#pragma unroll
      for (int gg = 0; gg < GROUPS; ++gg) {
        const float* pp = reinterpret_cast<const float*>(&part[gg][r][j / 4]);
        s += pp[j % 4];
      }
      if (r < kRows)
        a[r] = s;
      else
        bq[r - kRows] = s;
    }
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
      float pred = __expf(G[r]) * a[r];
      for (int s2 = 0; s2 < r; ++s2) pred += __expf(G[r] - G[s2]) * kk[s2][r] * delta[s2];
      delta[r] = bt[r] * (vr[r] - pred);
      float out = __expf(G[r]) * bq[r];
      for (int s2 = 0; s2 <= r; ++s2) out += __expf(G[r] - G[s2]) * kq[s2][r] * delta[s2];
      o[((row0 + r) * H_v + h) * D + j] = __bfloat16_as_ushort(__float2bfloat16_rn(scale * out));
      stash[size_t(b) * stash_seq_floats + size_t(h) * kRows * (D + 4) + r * D + j] = delta[r];
    }
  }
  if (tid < kRows)
    stash[size_t(b) * stash_seq_floats + size_t(h) * kRows * (D + 4) + kRows * D + tid] = G[tid];
}

// grid = (H_v, batch); block = 256.  Each thread loads all of its 16-byte
// state quads (16 at d = 128) before updating and storing them.
template <int D>
__global__ void __launch_bounds__(kVThreads) fold_kernel(float* const* __restrict__ h_table,
                                                         const float* __restrict__ stash,
                                                         const int32_t* __restrict__ na_tab,
                                                         const uint16_t* __restrict__ k,
                                                         int qk_stride, uint32_t* flag, int H_k,
                                                         int H_v, int stash_seq_floats) {
  constexpr int QUADS = D / 4;
  constexpr int PER = D * QUADS / kVThreads;  // quads per thread (16 resp. 4)
  __shared__ float ks[kRows][D], dl[kRows][D], coef[kRows], cdecay;
  const int h = blockIdx.x, b = blockIdx.y;
  const int tid = threadIdx.x;
  if ((*(volatile uint32_t*)flag & kFlagEngaged) == 0u) return;
  const int na = na_tab[b];
  float* H = h_table[b];
  if (na == 0 || H == nullptr) return;
  if (na < 0 || na > kRows) {
    if (h == 0 && tid == 0) atomicOr(flag, kFlagError);
    return;
  }
  float4* H4 = reinterpret_cast<float4*>(H + size_t(h) * D * D);
  float4 hv[PER];
#pragma unroll
  for (int m = 0; m < PER; ++m) hv[m] = H4[tid + kVThreads * m];
  const int hk = h / (H_v / H_k);
  const float* st = stash + size_t(b) * stash_seq_floats + size_t(h) * kRows * (D + 4);
  for (int idx = tid; idx < kRows * D; idx += kVThreads) {
    const int r = idx / D, i = idx % D;
    ks[r][i] = bf16_at(k + (size_t(b) * kRows + r) * qk_stride + size_t(hk) * D + i);
    dl[r][i] = st[r * D + i];
  }
  if (tid == 0) {
    const float Gl = st[kRows * D + na - 1];
    for (int r = 0; r < kRows; ++r) coef[r] = r < na ? __expf(Gl - st[kRows * D + r]) : 0.f;
    cdecay = __expf(Gl);
  }
  __syncthreads();
#pragma unroll
  for (int m = 0; m < PER; ++m) {
    const int idx = tid + kVThreads * m;
    const int i = idx / QUADS, j4 = idx % QUADS;
    float4 x = hv[m];
    x.x *= cdecay;
    x.y *= cdecay;
    x.z *= cdecay;
    x.w *= cdecay;
    for (int r = 0; r < na; ++r) {
      const float c = coef[r] * ks[r][i];
      x.x = fmaf(c, dl[r][4 * j4 + 0], x.x);
      x.y = fmaf(c, dl[r][4 * j4 + 1], x.y);
      x.z = fmaf(c, dl[r][4 * j4 + 2], x.z);
      x.w = fmaf(c, dl[r][4 * j4 + 3], x.w);
    }
    H4[idx] = x;
  }
}

cudaError_t launch_flag_clear(uint32_t* flag, cudaStream_t s) {
  flag_clear_kernel<<<1, 32, 0, s>>>(flag);
  return cudaGetLastError();
}

cudaError_t launch_verify(float* const* h_table, const uint16_t* q, const uint16_t* k,
                          int qk_stride, const uint16_t* v, int v_stride, const float* g,
                          const float* beta, int gb_stride, uint16_t* o, float* stash,
                          int stash_seq_floats, int batch, int H_k, int H_v, int D, float scale,
                          uint32_t* flag, cudaStream_t s) {
  if (batch == 0) return cudaSuccess;
  dim3 grid(H_v, batch);
  if (D == 128)
    verify_kernel<128><<<grid, kVThreads, 0, s>>>(h_table, q, k, qk_stride, v, v_stride, g, beta,
                                            gb_stride, o, stash, stash_seq_floats, H_k, H_v,
                                            scale, flag);
  else
    verify_kernel<64><<<grid, kVThreads, 0, s>>>(h_table, q, k, qk_stride, v, v_stride, g, beta,
                                           gb_stride, o, stash, stash_seq_floats, H_k, H_v,
                                           scale, flag);
  return cudaGetLastError();
}

cudaError_t launch_fold(float* const* h_table, const float* stash, const int32_t* na_tab,
                        const uint16_t* k, int qk_stride, uint32_t* flag, int k_rows, int batch,
                        int H_k, int H_v, int D, int stash_seq_floats, cudaStream_t s) {
  (void)k_rows;
  if (batch == 0) return cudaSuccess;
  dim3 grid(H_v, batch);
  if (D == 128)
    fold_kernel<128><<<grid, kVThreads, 0, s>>>(h_table, stash, na_tab, k, qk_stride, flag, H_k, H_v,
                                          stash_seq_floats);
  else
    fold_kernel<64><<<grid, kVThreads, 0, s>>>(h_table, stash, na_tab, k, qk_stride, flag, H_k, H_v,
                                         stash_seq_floats);
  return cudaGetLastError();
}

size_t static_stash_floats() { return kStaticStashFloats; }

// In host code g_static_stash names a host-side stand-in, not device memory,
// so its device address is looked up once per device (with that device
// current) and cached.
cudaError_t static_stash_address(float** out) {
  static std::mutex mu;
  static float* cache[64] = {nullptr};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (cache[dev] == nullptr) {
    float* ptr = nullptr;
    e = cudaGetSymbolAddress(reinterpret_cast<void**>(&ptr), g_static_stash);
    if (e != cudaSuccess) return e;
    cache[dev] = ptr;
  }
  *out = cache[dev];
  return cudaSuccess;
}

// Read and clear this file's device error word (host; synchronous).
cudaError_t take_err_verify(uint32_t* out) {
  uint32_t zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(out, g_err_verify, sizeof(uint32_t));
  if (e != cudaSuccess) return e;
  return cudaMemcpyToSymbol(g_err_verify, &zero, sizeof(uint32_t));
}

}  // namespace gdn
