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
// which is the token recurrence unrolled over four rows.  H0 is read once,
// streamed into shared memory by bulk copies (persistent kernel below);
// nothing is written to it.  delta_r and G_r go to the stash for the fold.
//
// Fold.  With na = na_tab[b] in 1..4 (and the engaged bit set):
//   H[i][j] <- e^{G_{na-1}} H[i][j] + sum_{r<na} e^{G_{na-1} - G_r} k_r[i] delta_r[j]
// reading and writing each state element once; na = 0 touches nothing.
// Parent (non write-on-accept) verify.  The same four rows, but the states are
// written: the state after row r, Hi(r), goes to the intermediate slab
// hi_tables[b * slab_entries + r] for r < 3 and the state after all four rows
// replaces the live state.  With the engaged word clear the fold then
// restores Hi(na - 1) into the live state on a partial accept (1 <= na < 4).
//
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
constexpr uint32_t kFlagStashBad = 4u;  // a verify gave up before its whole stash was written
constexpr int kRows = 4;

__device__ __forceinline__ float bf16_at(const uint16_t* p) {
  return __uint_as_float(uint32_t(*p) << 16);
}

__global__ void flag_clear_kernel(uint32_t* flag) {
  if (threadIdx.x == 0) *flag = 0u;
}

constexpr int kVThreads = 256;  // fold block

// ---------------------------------------------------------------------------
// Verify: one persistent CTA per SM walks the (sequence, v-head) items
// blockIdx.x, blockIdx.x + gridDim.x, ...  Warp roles, each warp running at
// its own pace (mbarriers only, no block-wide barrier inside the loop):
//   warps 0-7 (256 threads)  FMA: thread = (row group, column quad); reads
//       its rows of the item's state from shared memory and accumulates the
//       row-group partials of a_r and b_r for its four columns into part[];
//       warps 0-3 read the first half of the state, warps 4-7 the second.
//   warp 8   copies: each item's state, as two contiguous halves (rows
//       0 .. D/2 - 1 and D/2 .. D - 1), into a ring of shared-memory slots
//       with cp.async.bulk, as far ahead as the ring allows.
//   warps 9-11  item descriptors (warp 9 + m takes the items n = m mod 3 into
//       descriptor slot m): k and q transposed to 4-row vectors, v, the dot
//       products k_s.k_r and k_s.q_r, the cumulative gates and the decay
//       factors, prepared while earlier items compute (their global loads
//       take microseconds while the state copies saturate HBM, hence three).
//   warps 12-15  epilogue: thread j < D reduces the row groups of column j
//       and runs its 4-step recurrence, while the FMA warps go on with the
//       next item (part[] is double-buffered).
// ---------------------------------------------------------------------------
// Packed f32x2 arithmetic (two IEEE f32 FMAs per instruction): a pair lives
// in one 64-bit register, low half first.
__device__ __forceinline__ uint64_t dup_f32x2(float x) {
  uint64_t d;
  asm("mov.b64 %0, {%1, %1};" : "=l"(d) : "f"(x));
  return d;
}
__device__ __forceinline__ uint64_t fma_f32x2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ float lo_f32x2(uint64_t d) { return __uint_as_float(uint32_t(d)); }

// Shared-space loads by 32-bit shared address (the block's dynamic shared
// memory is addressed through a realigned generic pointer, which the
// compiler would otherwise access with generic loads).
__device__ __forceinline__ float4 lds_f4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr));
  return v;
}
__device__ __forceinline__ ulonglong2 lds_u64x2(uint32_t addr) {
  ulonglong2 v;
  asm volatile("ld.shared.v2.u64 {%0, %1}, [%2];" : "=l"(v.x), "=l"(v.y) : "r"(addr));
  return v;
}
__device__ __forceinline__ float lds_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr));
  return v;
}
__device__ __forceinline__ float hi_f32x2(uint64_t d) { return __uint_as_float(uint32_t(d >> 32)); }

constexpr int kVCompute = 256;
constexpr int kVCopyWarp = 8;
constexpr int kVDesc = 3;  // descriptor slots = descriptor warps (16 warps in all)
constexpr int kVEpiWarp = kVCopyWarp + 1 + kVDesc;
constexpr int kVEpi = 128;
constexpr int kVBlock = kVCompute + 32 * (1 + kVDesc) + kVEpi;
constexpr uint32_t kVRingBytes = 128 * 1024;

template <int D>
struct VerifyDesc {
  float4 kq[D][2];      // (k_0[i], q_0[i], k_1[i], q_1[i]), (k_2[i], q_2[i], k_3[i], q_3[i])
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
  static constexpr uint32_t PART_BYTES = uint32_t(GROUPS) * 2 * kRows * QUADS * 16;
  static constexpr uint32_t PART = 0 + kVRingBytes;  // 2 x float4 [GROUPS][2*kRows][QUADS]
  static constexpr uint32_t DESC = PART + 2 * PART_BYTES;
  static constexpr uint32_t BARS = DESC + kVDesc * uint32_t(sizeof(VerifyDesc<D>));
  // full[NSLOT], empty[NSLOT], dfull[kVDesc], dempty[kVDesc], pfull[2], pempty[2], abort word
  static constexpr uint32_t TOTAL = BARS + (2 * NSLOT + 2 * kVDesc + 4) * 8 + 16;
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
  // 128-byte aligned start, kept as an offset from the __shared__ array so
  // that accesses through it stay shared-space (not generic) loads and stores
  uint8_t* smem = smem_raw + ((uint32_t(128) - (smem_u32(smem_raw) & 127u)) & 127u);
  VerifyDesc<D>* desc = reinterpret_cast<VerifyDesc<D>*>(smem + L::DESC);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::BARS);
  uint64_t* empty = full + NSLOT;
  uint64_t* dfull = empty + NSLOT;
  uint64_t* dempty = dfull + kVDesc;
  uint64_t* pfull = dempty + kVDesc;
  uint64_t* pempty = pfull + 2;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(pempty + 2);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int items = batch * H_v;
  const int vpg = H_v / H_k;
  if (tid == 0) {
    for (int i = 0; i < NSLOT; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 4);  // the four warps that read a half
    }
    for (int i = 0; i < kVDesc; ++i) {
      mbar_init(&dfull[i], 32);
      mbar_init(&dempty[i], (kVCompute + kVEpi) / 32);  // FMA and epilogue warps
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&pfull[i], kVCompute / 32);
      mbar_init(&pempty[i], kVEpi / 32);
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
  } else if (warp > kVCopyWarp && warp < kVEpiWarp) {
    // ---------------- item descriptors: warp 9 + m the items n = m (mod kVDesc)
    const int ds = warp - kVCopyWarp - 1;
    int n = ds;
    for (int it = blockIdx.x + ds * gridDim.x; it < items; it += kVDesc * gridDim.x, n += kVDesc) {
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
      const int use = n / kVDesc;
      bool ok = use == 0 || mbar_wait(&dempty[ds], (use - 1) & 1, abort_flag, &g_err_verify, 2u);
      if (!__all_sync(0xffffffffu, ok)) break;
      VerifyDesc<D>& d = desc[ds];
      if (!pad) {
#pragma unroll
        for (int e = 0; e < EPL; ++e) {
          const int i = lane + 32 * e;
          d.kq[i][0] = make_float4(kr[0][e], qr[0][e], kr[1][e], qr[1][e]);
          d.kq[i][1] = make_float4(kr[2][e], qr[2][e], kr[3][e], qr[3][e]);
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
        // every lane holds the totals and the cumulative gates; lane
        // 4 s + r writes the [s][r] factors, lanes r < 4 the per-row ones
        float Gc[kRows];
        float run = 0.f;
#pragma unroll
        for (int r = 0; r < kRows; ++r) {
          run += gr[r];
          Gc[r] = run;
        }
        if (lane < kRows * kRows) {
          const int s2 = lane >> 2, r = lane & 3;
          float gs = Gc[0], grr = Gc[0], kkv = dk[0][0], kqv = dq[0][0];
#pragma unroll
          for (int x = 0; x < kRows; ++x) {
            if (x == s2) gs = Gc[x];
            if (x == r) grr = Gc[x];
#pragma unroll
            for (int y = 0; y < kRows; ++y)
              if (x == s2 && y == r) {
                kkv = dk[x][y];
                kqv = dq[x][y];
              }
          }
          const float e = __expf(grr - gs);
          d.cK[s2][r] = s2 < r ? e * kkv : 0.f;
          d.cQ[s2][r] = s2 <= r ? e * kqv : 0.f;
          if (lane < kRows) {
            float gl = Gc[0], bl = br[0];
#pragma unroll
            for (int x = 1; x < kRows; ++x)
              if (x == lane) {
                gl = Gc[x];
                bl = br[x];
              }
            d.eG[lane] = __expf(gl);
            d.bt[lane] = bl;
            d.Gc[lane] = gl;
          }
        }
      }
      if (lane == 0) d.pad = pad ? 1 : 0;
      mbar_arrive(&dfull[ds]);  // every lane, after its own writes
    }
  } else if (warp < kVCopyWarp) {
    // ---------------- FMA warps (256 threads)
    const int quad = tid % QUADS, grp = tid / QUADS;
    const int half = grp / (GROUPS / 2);
    const int lrow0 = (grp - half * (GROUPS / 2)) * RPG;  // first row within the half
    int sc = 0, n = 0;
    bool ok = true;
    for (int it = blockIdx.x; it < items && ok; it += gridDim.x, ++n) {
      const int ds = n % kVDesc, pb = n & 1, pu = n >> 1;
      ok = mbar_wait(&dfull[ds], (n / kVDesc) & 1, abort_flag, &g_err_verify, 4u);
      if (!__all_sync(0xffffffffu, ok)) break;
      const VerifyDesc<D>& d = desc[ds];
      const bool pad = d.pad != 0;
      // acc[c][r] = (a_r, b_r) partials of column 4 quad + c
      uint64_t acc[4][kRows];
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int r = 0; r < kRows; ++r) acc[c][r] = 0ull;
      if (!pad) {
        const int c = sc + half;
        const int slot = c % NSLOT;
        ok = mbar_wait(&full[slot], (c / NSLOT) & 1, abort_flag, &g_err_verify, 4u);
        if (ok) {
          const uint32_t s_row = smem_u32(smem + size_t(slot) * L::HALF) +
                                 uint32_t((lrow0 * QUADS + quad) * 16);
          const uint32_t kq_row = smem_u32(&d.kq[grp * RPG][0]);
#pragma unroll 4
          for (int ii = 0; ii < RPG; ++ii) {
            const float4 hv = lds_f4(s_row + uint32_t(ii * QUADS * 16));
            const ulonglong2 p01 = lds_u64x2(kq_row + uint32_t(ii * 32));
            const ulonglong2 p23 = lds_u64x2(kq_row + uint32_t(ii * 32 + 16));
            const uint64_t kq2[kRows] = {p01.x, p01.y, p23.x, p23.y};  // (k_r[i], q_r[i])
            const float hs[4] = {hv.x, hv.y, hv.z, hv.w};
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
              const uint64_t s2 = dup_f32x2(hs[cc]);
#pragma unroll
              for (int r = 0; r < kRows; ++r) acc[cc][r] = fma_f32x2(s2, kq2[r], acc[cc][r]);
            }
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[slot]);  // this warp is done with the slot
        sc += 2;
        if (!__all_sync(0xffffffffu, ok)) break;
      }
      // part[pb] is free once the epilogue finished item n - 2
      ok = pu == 0 || mbar_wait(&pempty[pb], (pu - 1) & 1, abort_flag, &g_err_verify, 4u);
      if (!__all_sync(0xffffffffu, ok)) break;
      if (!pad) {
        const uint32_t part = smem_u32(smem + L::PART + pb * L::PART_BYTES);
#pragma unroll
        for (int r = 0; r < kRows; ++r) {
          st_shared_v4(part + uint32_t(((grp * 2 * kRows + r) * QUADS + quad) * 16),
                       uint32_t(acc[0][r]), uint32_t(acc[1][r]), uint32_t(acc[2][r]),
                       uint32_t(acc[3][r]));
          st_shared_v4(part + uint32_t(((grp * 2 * kRows + kRows + r) * QUADS + quad) * 16),
                       uint32_t(acc[0][r] >> 32), uint32_t(acc[1][r] >> 32),
                       uint32_t(acc[2][r] >> 32), uint32_t(acc[3][r] >> 32));
        }
      }
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&pfull[pb]);
        mbar_arrive(&dempty[ds]);  // the FMA warps are done with the descriptor
      }
    }
    if (!ok) *abort_flag = 1;
  } else {
    // ---------------- epilogue warps (128 threads): reduction + recurrence
    const int et = tid - kVEpiWarp * 32;
    int n = 0;
    bool ok = true;
    for (int it = blockIdx.x; it < items && ok; it += gridDim.x, ++n) {
      const int b = it / H_v, h = it - b * H_v;
      const int ds = n % kVDesc, pb = n & 1;
      ok = mbar_wait(&dfull[ds], (n / kVDesc) & 1, abort_flag, &g_err_verify, 8u) &&
           mbar_wait(&pfull[pb], (n >> 1) & 1, abort_flag, &g_err_verify, 8u);
      if (!__all_sync(0xffffffffu, ok)) break;
      const VerifyDesc<D>& d = desc[ds];
      if (et < D) {
        const int j = et;
        const size_t row0 = size_t(b) * kRows;
        if (d.pad != 0) {
#pragma unroll
          for (int r = 0; r < kRows; ++r) o[((row0 + r) * H_v + h) * D + j] = 0;
        } else {
          const uint32_t pf = smem_u32(smem + L::PART + pb * L::PART_BYTES) + uint32_t(j * 4);
          float a[kRows], bq[kRows], delta[kRows];
#pragma unroll
          for (int r = 0; r < 2 * kRows; ++r) {
            float s2 = 0.f;
#pragma unroll
            for (int gg = 0; gg < GROUPS; ++gg) s2 += lds_f32(pf + uint32_t((gg * 2 * kRows + r) * D * 4));
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
      if (lane == 0) {
        mbar_arrive(&pempty[pb]);
        mbar_arrive(&dempty[ds]);  // the epilogue warps are done with the descriptor
      }
    }
    if (!ok) *abort_flag = 1;
  }
  __syncthreads();
  // A CTA that gave up (a bounded wait ran out) left part of its stash
  // unwritten: say so in the engaged word, so that the fold applies nothing.
  if (tid == 0 && *abort_flag) atomicOr(flag, kFlagError | kFlagStashBad);
}

// grid = (H_v, batch); block = 256.  Each thread loads all of its 16-byte
// state quads (16 at d = 128) before updating and storing them.
template <int D>
__global__ void __launch_bounds__(kVThreads) fold_kernel(float* const* __restrict__ h_table,
                                                         const float* __restrict__ stash,
                                                         const int32_t* __restrict__ na_tab,
                                                         const uint16_t* __restrict__ k,
                                                         int qk_stride,
                                                         float* const* __restrict__ hi_tables,
                                                         int slab_entries, uint32_t* flag,
                                                         int H_k, int H_v, int stash_seq_floats) {
  constexpr int QUADS = D / 4;
  constexpr int PER = D * QUADS / kVThreads;  // quads per thread (16 resp. 4)
  __shared__ float ks[kRows][D], dl[kRows][D], coef[kRows], cdecay;
  const int h = blockIdx.x, b = blockIdx.y;
  const int tid = threadIdx.x;
  const uint32_t fw = *(volatile uint32_t*)flag;
  const int na = na_tab[b];
  float* H = h_table[b];
  if ((fw & kFlagEngaged) == 0u) {
    // The parent verify ran: the live state holds the state after all four
    // rows; a partial accept restores the kept intermediate Hi(na - 1).
    if (hi_tables == nullptr || H == nullptr || na == kRows) return;
    const float* src =
        (na >= 1 && na < kRows) ? hi_tables[size_t(b) * slab_entries + (na - 1)] : nullptr;
    if (src == nullptr) {  // na out of range (0 included: the pre-verify state is gone)
      if (h == 0 && tid == 0) atomicOr(flag, kFlagError);
      return;
    }
    const float4* s4 = reinterpret_cast<const float4*>(src + size_t(h) * D * D);
    float4* d4 = reinterpret_cast<float4*>(H + size_t(h) * D * D);
    float4 hv[PER];
#pragma unroll
    for (int m = 0; m < PER; ++m) hv[m] = s4[tid + kVThreads * m];
#pragma unroll
    for (int m = 0; m < PER; ++m) d4[tid + kVThreads * m] = hv[m];
    return;
  }
  if ((fw & kFlagStashBad) != 0u) return;
  if (na == 0 || H == nullptr) return;
  if (na < 0 || na > kRows || stash == nullptr || k == nullptr) {
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

// ---------------------------------------------------------------------------
// Parent verify: grid = (H_v, batch), 256 threads, one (sequence, v-head) item
// per CTA.  Pass 1 reduces the state columns against the four k and q rows
// (thread = (column j, row slice)); thread j < D then runs the 4-step column
// recurrence of the header (o rows and delta rows); pass 2 writes Hi(0..2) to
// the slabs and Hi(3) over the live state, each element
//   Hi(r)[i][j] = e^{G_r} H0[i][j] + sum_{s<=r} e^{G_r - G_s} k_s[i] delta_s[j],
// re-reading H0 (from L2) as 16-byte quads.  No waits: nothing can hang.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) verify_parent_kernel(
    float* const* __restrict__ h_table, const uint16_t* __restrict__ q,
    const uint16_t* __restrict__ k, int qk_stride, const uint16_t* __restrict__ v, int v_stride,
    const float* __restrict__ g, const float* __restrict__ beta, int gb_stride,
    uint16_t* __restrict__ o, float* const* __restrict__ hi_tables, int slab_entries, int H_k,
    int H_v, float scale) {
  constexpr int NT = 256, QUADS = D / 4, SLICES = NT / D, RPS = D / SLICES;
  __shared__ float ks[kRows][D], qs[kRows][D], dl[kRows][D];
  __shared__ float part[SLICES][2 * kRows][D];
  __shared__ float cK[kRows][kRows], cQ[kRows][kRows], cf[kRows][kRows];
  __shared__ float eG[kRows], bt[kRows], Gc[kRows];
  const int h = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int hk = h / (H_v / H_k);
  float* live = h_table[b];
  const size_t row0 = size_t(b) * kRows;
  if (live == nullptr) {  // padding sequence: zero outputs, no state
    for (int idx = tid; idx < kRows * D; idx += NT) {
      const int r = idx / D, j = idx % D;
      o[((row0 + r) * H_v + h) * D + j] = 0;
    }
    return;
  }
  const float* H0 = live + size_t(h) * D * D;
  for (int idx = tid; idx < kRows * D; idx += NT) {
    const int r = idx / D, i = idx % D;
    ks[r][i] = bf16_at(k + (row0 + r) * qk_stride + size_t(hk) * D + i);
    qs[r][i] = bf16_at(q + (row0 + r) * qk_stride + size_t(hk) * D + i);
  }
  __syncthreads();
  // k_s . k_r and k_s . q_r: warp w takes the four products 4 w .. 4 w + 3
  // (the first 16 are k.k, the next 16 k.q); the gates on the side
  for (int m = 0; m < 4; ++m) {
    const int pidx = 4 * warp + m, sr = pidx & 15, s2 = sr >> 2, r = sr & 3;
    const float* other = pidx < 16 ? ks[r] : qs[r];
    float acc = 0.f;
    for (int i = lane; i < D; i += 32) acc = fmaf(ks[s2][i], other[i], acc);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (lane == 0) {
      if (pidx < 16)
        cK[s2][r] = acc;
      else
        cQ[s2][r] = acc;
    }
  }
  if (tid == 0) {
    float run = 0.f;
    for (int r = 0; r < kRows; ++r) {
      run += g[(row0 + r) * gb_stride + h];
      Gc[r] = run;
      bt[r] = beta[(row0 + r) * gb_stride + h];
      eG[r] = __expf(run);
    }
  }
  // pass 1: column partials a_r[j] = sum_i H0[i][j] k_r[i], b_r[j] likewise with q_r
  {
    const int j = tid % D, sl = tid / D;
    float a[kRows] = {0.f, 0.f, 0.f, 0.f}, bq[kRows] = {0.f, 0.f, 0.f, 0.f};
    for (int ii = 0; ii < RPS; ++ii) {
      const int i = sl * RPS + ii;
      const float hv = H0[size_t(i) * D + j];
#pragma unroll
      for (int r = 0; r < kRows; ++r) {
        a[r] = fmaf(hv, ks[r][i], a[r]);
        bq[r] = fmaf(hv, qs[r][i], bq[r]);
      }
    }
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
      part[sl][r][j] = a[r];
      part[sl][kRows + r][j] = bq[r];
    }
  }
  __syncthreads();
  if (tid == 0) {  // decay factors of the pair products (scalars, once)
    for (int s2 = 0; s2 < kRows; ++s2)
      for (int r = 0; r < kRows; ++r) {
        const float e = __expf(Gc[r] - Gc[s2]);
        cK[s2][r] = s2 < r ? e * cK[s2][r] : 0.f;
        cQ[s2][r] = s2 <= r ? e * cQ[s2][r] : 0.f;
        cf[r][s2] = s2 <= r ? e : 0.f;
      }
  }
  __syncthreads();
  if (tid < D) {
    const int j = tid;
    float a[kRows], bq[kRows], delta[kRows];
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
      float x = 0.f, y = 0.f;
#pragma unroll
      for (int sl = 0; sl < SLICES; ++sl) {
        x += part[sl][r][j];
        y += part[sl][kRows + r][j];
      }
      a[r] = x;
      bq[r] = y;
    }
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
      float pred = eG[r] * a[r];
#pragma unroll
      for (int s2 = 0; s2 < r; ++s2) pred += cK[s2][r] * delta[s2];
      delta[r] = bt[r] * (bf16_at(v + (row0 + r) * v_stride + size_t(h) * D + j) - pred);
      float out = eG[r] * bq[r];
#pragma unroll
      for (int s2 = 0; s2 <= r; ++s2) out += cQ[s2][r] * delta[s2];
      o[((row0 + r) * H_v + h) * D + j] = __bfloat16_as_ushort(__float2bfloat16_rn(scale * out));
      dl[r][j] = delta[r];
    }
  }
  __syncthreads();
  // pass 2: the four states; the live state is written last (H0 is re-read
  // from it until then, and every read of a quad precedes its own write)
  float* dst[kRows];
#pragma unroll
  for (int r = 0; r < kRows - 1; ++r)
    dst[r] = hi_tables != nullptr ? hi_tables[size_t(b) * slab_entries + r] : nullptr;
  dst[kRows - 1] = live;
  const float4* H04 = reinterpret_cast<const float4*>(H0);
  for (int idx = tid; idx < D * QUADS; idx += NT) {
    const int i = idx / QUADS, j4 = idx % QUADS;
    const float4 h0v = H04[idx];
    float kv[kRows];
#pragma unroll
    for (int s2 = 0; s2 < kRows; ++s2) kv[s2] = ks[s2][i];
    float4 out[kRows];
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
      float x0 = eG[r] * h0v.x, x1 = eG[r] * h0v.y, x2 = eG[r] * h0v.z, x3 = eG[r] * h0v.w;
#pragma unroll
      for (int s2 = 0; s2 <= r; ++s2) {
        const float c = cf[r][s2] * kv[s2];
        x0 = fmaf(c, dl[s2][4 * j4 + 0], x0);
        x1 = fmaf(c, dl[s2][4 * j4 + 1], x1);
        x2 = fmaf(c, dl[s2][4 * j4 + 2], x2);
        x3 = fmaf(c, dl[s2][4 * j4 + 3], x3);
      }
      out[r] = make_float4(x0, x1, x2, x3);
    }
#pragma unroll
    for (int r = 0; r < kRows; ++r)
      if (dst[r] != nullptr)
        reinterpret_cast<float4*>(dst[r] + size_t(h) * D * D)[idx] = out[r];
  }
}

cudaError_t launch_verify_parent(float* const* h_table, const uint16_t* q, const uint16_t* k,
                                 int qk_stride, const uint16_t* v, int v_stride, const float* g,
                                 const float* beta, int gb_stride, uint16_t* o,
                                 float* const* hi_tables, int slab_entries, int batch, int H_k,
                                 int H_v, int D, float scale, cudaStream_t s) {
  if (batch == 0) return cudaSuccess;
  dim3 grid(H_v, batch);
  if (D == 128)
    verify_parent_kernel<128><<<grid, 256, 0, s>>>(h_table, q, k, qk_stride, v, v_stride, g,
                                                   beta, gb_stride, o, hi_tables, slab_entries,
                                                   H_k, H_v, scale);
  else
    verify_parent_kernel<64><<<grid, 256, 0, s>>>(h_table, q, k, qk_stride, v, v_stride, g, beta,
                                                  gb_stride, o, hi_tables, slab_entries, H_k,
                                                  H_v, scale);
  return cudaGetLastError();
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
                        const uint16_t* k, int qk_stride, float* const* hi_tables,
                        int slab_entries, uint32_t* flag, int k_rows, int batch, int H_k, int H_v,
                        int D, int stash_seq_floats, cudaStream_t s) {
  (void)k_rows;
  if (batch == 0) return cudaSuccess;
  dim3 grid(H_v, batch);
  if (D == 128)
    fold_kernel<128><<<grid, kVThreads, 0, s>>>(h_table, stash, na_tab, k, qk_stride, hi_tables,
                                                slab_entries, flag, H_k, H_v, stash_seq_floats);
  else
    fold_kernel<64><<<grid, kVThreads, 0, s>>>(h_table, stash, na_tab, k, qk_stride, hi_tables,
                                               slab_entries, flag, H_k, H_v, stash_seq_floats);
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
