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

constexpr int kVThreads = 256;  // fold block; verify compute threads

// ---------------------------------------------------------------------------
// Verify: one persistent CTA per SM walks the (sequence, v-head) items
// blockIdx.x, blockIdx.x + gridDim.x, ...  Warp roles:
//   warps 0-7 (256 threads)  compute: thread = (row group, column quad); the
//       FMA phase reads its rows of the item's state from shared memory and
//       accumulates a_r and b_r for its four columns; warps 0 .. D/32 - 1 then
//       reduce the row groups and run the per-column 4-step recurrence.
//   warp 8   copies: each item's state, as two contiguous halves (rows
//       0 .. D/2 - 1 and D/2 .. D - 1), into a ring of shared-memory slots
//       with cp.async.bulk, as far ahead as the ring allows.
//   warps 9, 10  item descriptors (even / odd items): k and q transposed to
//       4-row vectors, v, the dot products k_s.k_r and k_s.q_r, the cumulative
//       gates and the decay factors, prepared while earlier items compute.
// Warps 0-3 read the first half of the state, warps 4-7 the second.
// ---------------------------------------------------------------------------
constexpr int kVCompute = 256;
constexpr int kVCopyWarp = 8;
constexpr int kVBlock = kVCompute + 3 * 32;
constexpr uint32_t kVRingBytes = 160 * 1024;

template <int D>
struct VerifyDesc {
  float4 kq4[D];        // (k_0[i], k_1[i], k_2[i], k_3[i])
  float4 qq4[D];        // (q_0[i], .., q_3[i])
  float vv[kRows][D];   // v rows
  float eG[kRows];      // e^{G_r}
  float cK[kRows][kRows];  // [s][r] = e^{G_r - G_s} k_s.k_r   (s < r)
  float cQ[kRows][kRows];  // [s][r] = e^{G_r - G_s} k_s.q_r   (s <= r)
  float bt[kRows];      // beta_r
  float Gc[kRows];      // G_r (stashed for the fold)
  int pad;              // 1: the sequence has no state (zero outputs only)
  int pad_[3];
};

template <int D>
struct VerifySmem {
  static constexpr int QUADS = D / 4;
  static constexpr int GROUPS = kVCompute / QUADS;  // 8 (D=128) / 16 (D=64)
  static constexpr int RPG = D / GROUPS;            // rows per group: 16 / 4
  static constexpr uint32_t HALF = uint32_t(D) * D * 4 / 2;
  static constexpr int NSLOT = int(kVRingBytes / HALF);
  static constexpr uint32_t PART = 0 + kVRingBytes;  // float4 [GROUPS][2*kRows][QUADS]
  static constexpr uint32_t DESC = PART + uint32_t(GROUPS) * 2 * kRows * QUADS * 16;
  static constexpr uint32_t BARS = DESC + 2 * uint32_t(sizeof(VerifyDesc<D>));
  // full[NSLOT], empty[NSLOT], dfull[2], dempty[2], abort word
  static constexpr uint32_t TOTAL = BARS + (2 * NSLOT + 4) * 8 + 16;
};
static_assert(VerifySmem<128>::TOTAL + 128 <= 232448, "verify shared memory");
static_assert(VerifySmem<64>::TOTAL + 128 <= 232448, "verify shared memory");

template <int D>
__global__ void __launch_bounds__(kVBlock, 1) verify_kernel(
    float* const* __restrict__ h_table, const uint16_t* __restrict__ q,
    const uint16_t* __restrict__ k, int qk_stride, const uint16_t* __restrict__ v, int v_stride,
    const float* __restrict__ g, const float* __restrict__ beta, int gb_stride,
    uint16_t* __restrict__ o, float* __restrict__ stash, int stash_seq_floats, int batch, int H_k,
    int H_v, float scale, uint32_t* flag) {
  using L = VerifySmem<D>;
  constexpr int QUADS = L::QUADS, GROUPS = L::GROUPS, RPG = L::RPG, NSLOT = L::NSLOT;
  constexpr int EPL = D / 32;  // elements of a row per lane (descriptor warps)
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) &
                                             ~uintptr_t(127));
  float4* part = reinterpret_cast<float4*>(smem + L::PART);
  VerifyDesc<D>* desc = reinterpret_cast<VerifyDesc<D>*>(smem + L::DESC);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::BARS);
  uint64_t* empty = full + NSLOT;
  uint64_t* dfull = empty + NSLOT;
  uint64_t* dempty = dfull + 2;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(dempty + 2);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int items = batch * H_v;
  const int vpg = H_v / H_k;
  if (tid == 0) {
    for (int i = 0; i < NSLOT; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 4);  // the four warps that read a half
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&dfull[i], 32);
      mbar_init(&dempty[i], kVCompute / 32);
    }
    *abort_flag = 0;
    fence_barrier_init();
    if (blockIdx.x == 0) atomicOr(flag, kFlagEngaged);
  }
  __syncthreads();

  if (warp == kVCopyWarp) {
    // ---------------- state copies: two halves per item with a state
    if (lane == 0) {
      int sc = 0;
      bool ok = true;
      for (int it = blockIdx.x; it < items && ok; it += gridDim.x) {
        const int b = it / H_v, h = it - b * H_v;
        const float* H0 = h_table[b];
        if (H0 == nullptr) continue;
        for (int hf = 0; hf < 2 && ok; ++hf, ++sc) {
          const int slot = sc % NSLOT, use = sc / NSLOT;
          if (use > 0) ok = mbar_wait(&empty[slot], (use - 1) & 1, abort_flag, &g_err_verify, 1u);
          if (!ok) break;
          mbar_arrive_expect_tx(&full[slot], L::HALF);
          bulk_load_g2s(smem + size_t(slot) * L::HALF,
                        H0 + size_t(h) * D * D + size_t(hf) * (D / 2) * D, L::HALF, &full[slot]);
        }
      }
      if (!ok) *abort_flag = 1;
      // nothing may still be landing in shared memory at exit
      for (int c = max(0, sc - NSLOT); c < sc; ++c)
        mbar_wait(&full[c % NSLOT], (c / NSLOT) & 1, nullptr, &g_err_verify, 1u);
    }
    __syncwarp();
  } else if (warp > kVCopyWarp) {
    // ---------------- item descriptors: warp 9 the even, warp 10 the odd items
    const int ds = warp - kVCopyWarp - 1;
    int n = ds;
    for (int it = blockIdx.x + ds * gridDim.x; it < items; it += 2 * gridDim.x, n += 2) {
      const int b = it / H_v, h = it - b * H_v;
      const int hk = h / vpg;
      const bool pad = h_table[b] == nullptr;
      // raw rows into registers before the slot is free: lane l takes i = l + 32 e
      float kr[kRows][EPL], qr[kRows][EPL], vr[kRows][EPL], gr[kRows], br[kRows];
      if (!pad) {
#pragma unroll
        for (int r = 0; r < kRows; ++r) {
          const size_t row = size_t(b) * kRows + r;
#pragma unroll
          for (int e = 0; e < EPL; ++e) {
            const int i = lane + 32 * e;
            kr[r][e] = bf16_at(k + row * qk_stride + size_t(hk) * D + i);
            qr[r][e] = bf16_at(q + row * qk_stride + size_t(hk) * D + i);
            vr[r][e] = bf16_at(v + row * v_stride + size_t(h) * D + i);
          }
          gr[r] = g[row * gb_stride + h];
          br[r] = beta[row * gb_stride + h];
        }
      }
      const int use = n >> 1;
      bool ok = use == 0 || mbar_wait(&dempty[ds], (use - 1) & 1, abort_flag, &g_err_verify, 2u);
      if (!__all_sync(0xffffffffu, ok)) break;
      VerifyDesc<D>& d = desc[ds];
      if (!pad) {
#pragma unroll
        for (int e = 0; e < EPL; ++e) {
          const int i = lane + 32 * e;
          d.kq4[i] = make_float4(kr[0][e], kr[1][e], kr[2][e], kr[3][e]);
          d.qq4[i] = make_float4(qr[0][e], qr[1][e], qr[2][e], qr[3][e]);
#pragma unroll
          for (int r = 0; r < kRows; ++r) d.vv[r][i] = vr[r][e];
        }
        // k_s.k_r and k_s.q_r: lane partials, then a butterfly over the warp
        float dk[kRows][kRows], dq[kRows][kRows];
#pragma unroll
        for (int s2 = 0; s2 < kRows; ++s2)
#pragma unroll
          for (int r = 0; r < kRows; ++r) {
            float a = 0.f, c = 0.f;
#pragma unroll
            for (int e = 0; e < EPL; ++e) {
              a = fmaf(kr[s2][e], kr[r][e], a);
              c = fmaf(kr[s2][e], qr[r][e], c);
            }
            dk[s2][r] = a;
            dq[s2][r] = c;
          }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1)
#pragma unroll
          for (int s2 = 0; s2 < kRows; ++s2)
#pragma unroll
            for (int r = 0; r < kRows; ++r) {
              dk[s2][r] += __shfl_xor_sync(0xffffffffu, dk[s2][r], off);
              dq[s2][r] += __shfl_xor_sync(0xffffffffu, dq[s2][r], off);
            }
        if (lane == 0) {
          float Gc[kRows];
          float run = 0.f;
#pragma unroll
          for (int r = 0; r < kRows; ++r) {
            run += gr[r];
            Gc[r] = run;
          }
#pragma unroll
          for (int r = 0; r < kRows; ++r) {
            d.eG[r] = __expf(Gc[r]);
            d.bt[r] = br[r];
            d.Gc[r] = Gc[r];
#pragma unroll
            for (int s2 = 0; s2 < kRows; ++s2) {
              const float e = __expf(Gc[r] - Gc[s2]);
              d.cK[s2][r] = s2 < r ? e * dk[s2][r] : 0.f;
              d.cQ[s2][r] = s2 <= r ? e * dq[s2][r] : 0.f;
            }
          }
        }
      }
      if (lane == 0) d.pad = pad ? 1 : 0;
      mbar_arrive(&dfull[ds]);  // every lane, after its own writes
    }
  } else {
    // ---------------- compute (256 threads)
    const int quad = tid % QUADS, grp = tid / QUADS;
    const int half = grp / (GROUPS / 2);
    const int lrow0 = (grp - half * (GROUPS / 2)) * RPG;  // first row within the half
    int sc = 0, n = 0;
    for (int it = blockIdx.x; it < items; it += gridDim.x, ++n) {
      const int b = it / H_v, h = it - b * H_v;
      const int ds = n & 1;
      bool ok = mbar_wait(&dfull[ds], (n >> 1) & 1, abort_flag, &g_err_verify, 4u);
      const VerifyDesc<D>& d = desc[ds];
      const bool pad = ok && d.pad != 0;
      float4 acc[2 * kRows];
#pragma unroll
      for (int r = 0; r < 2 * kRows; ++r) acc[r] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (ok && !pad) {
        const int c = sc + half;
        const int slot = c % NSLOT;
        ok = mbar_wait(&full[slot], (c / NSLOT) & 1, abort_flag, &g_err_verify, 4u);
        if (ok) {
          const float4* S4 = reinterpret_cast<const float4*>(smem + size_t(slot) * L::HALF);
#pragma unroll 4
          for (int ii = 0; ii < RPG; ++ii) {
            const int i = grp * RPG + ii;
            const float4 hv = S4[(lrow0 + ii) * QUADS + quad];
            const float4 kv = d.kq4[i], qv = d.qq4[i];
            const float kk4[kRows] = {kv.x, kv.y, kv.z, kv.w};
            const float qq4[kRows] = {qv.x, qv.y, qv.z, qv.w};
#pragma unroll
            for (int r = 0; r < kRows; ++r) {
              acc[r].x = fmaf(hv.x, kk4[r], acc[r].x);
              acc[r].y = fmaf(hv.y, kk4[r], acc[r].y);
              acc[r].z = fmaf(hv.z, kk4[r], acc[r].z);
              acc[r].w = fmaf(hv.w, kk4[r], acc[r].w);
              acc[kRows + r].x = fmaf(hv.x, qq4[r], acc[kRows + r].x);
              acc[kRows + r].y = fmaf(hv.y, qq4[r], acc[kRows + r].y);
              acc[kRows + r].z = fmaf(hv.z, qq4[r], acc[kRows + r].z);
              acc[kRows + r].w = fmaf(hv.w, qq4[r], acc[kRows + r].w);
            }
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[slot]);  // this warp is done with the slot
        sc += 2;
      }
      // every compute thread agrees before going on (the previous item's
      // reduction has also finished reading part[])
      if (!named_all(1, kVCompute, ok)) {
        *abort_flag = 1;
        break;
      }
      if (!pad) {
#pragma unroll
        for (int r = 0; r < 2 * kRows; ++r) part[(grp * 2 * kRows + r) * QUADS + quad] = acc[r];
      }
      named_sync(2, kVCompute);
      if (tid < D) {
        const int j = tid;
        const size_t row0 = size_t(b) * kRows;
        if (pad) {
#pragma unroll
          for (int r = 0; r < kRows; ++r) o[((row0 + r) * H_v + h) * D + j] = 0;
        } else {
          const float* pf = reinterpret_cast<const float*>(part);
          float a[kRows], bq[kRows], delta[kRows];
#pragma unroll
          for (int r = 0; r < 2 * kRows; ++r) {
            float s2 = 0.f;
#pragma unroll
            for (int gg = 0; gg < GROUPS; ++gg) s2 += pf[(gg * 2 * kRows + r) * D + j];
            if (r < kRows)
              a[r] = s2;
            else
              bq[r - kRows] = s2;
          }
          float* st = stash + size_t(b) * stash_seq_floats + size_t(h) * kRows * (D + 4);
#pragma unroll
          for (int r = 0; r < kRows; ++r) {
            float pred = d.eG[r] * a[r];
#pragma unroll
            for (int s2 = 0; s2 < r; ++s2) pred += d.cK[s2][r] * delta[s2];
            delta[r] = d.bt[r] * (d.vv[r][j] - pred);
            float out = d.eG[r] * bq[r];
#pragma unroll
            for (int s2 = 0; s2 <= r; ++s2) out += d.cQ[s2][r] * delta[s2];
            o[((row0 + r) * H_v + h) * D + j] = __bfloat16_as_ushort(__float2bfloat16_rn(scale * out));
            st[r * D + j] = delta[r];
          }
          if (j < kRows) st[kRows * D + j] = d.Gc[j];
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&dempty[ds]);  // this warp is done with the descriptor
    }
  }
  __syncthreads();
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
  const int items = batch * H_v;
  const int grid = items < sm_count() ? items : sm_count();
  if (D == 128) {
    const int smem = int(VerifySmem<128>::TOTAL) + 128;
    cudaError_t e = cudaFuncSetAttribute(verify_kernel<128>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    verify_kernel<128><<<grid, kVBlock, smem, s>>>(h_table, q, k, qk_stride, v, v_stride, g,
                                                   beta, gb_stride, o, stash, stash_seq_floats,
                                                   batch, H_k, H_v, scale, flag);
  } else {
    const int smem = int(VerifySmem<64>::TOTAL) + 128;
    cudaError_t e = cudaFuncSetAttribute(verify_kernel<64>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    verify_kernel<64><<<grid, kVBlock, smem, s>>>(h_table, q, k, qk_stride, v, v_stride, g,
                                                  beta, gb_stride, o, stash, stash_seq_floats,
                                                  batch, H_k, H_v, scale, flag);
  }
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
