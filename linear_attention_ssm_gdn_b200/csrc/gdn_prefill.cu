// gdn_prefill.cu -- chunk-parallel gated delta rule prefill on sm_100a.
//
// Page "ssm_gdn_tc_route.rs" names the piece this file replaces: the prefill
// "state spine" (chunk_delta_h) that carries the f32 recurrent state H across
// chunks with bf16 tensor-core operands and an f32 accumulator.  Here the whole
// chunk step is fused into one kernel: per (sequence, v-head) unit one CTA
// walks the chunks (C = 64 rows) of its sequence, H stays on chip in f32 for
// the whole walk, and every contraction runs on tcgen05 with TMEM accumulators.
//
// Per chunk (rows r, s < 64; G_r = g_0 + ... + g_r; Gamma[r][s] = e^{G_r-G_s}):
//   P1 = [K;Q] K^T                                     (MMA, M=128 N=64 K=d_k)
//   A[r][s]   = beta_r Gamma[r][s] (k_r.k_s),  s < r   (prep warps, f32)
//   Aqk[r][s] = scale Gamma[r][s] (q_r.k_s),   s <= r
//   T  = (I + A)^{-1}                                  (blocked, f32)
//   T1 = T diag(beta e^G),  T2 = T diag(beta)
//   W^T = K^T T1^T   -> smem (bf16)                    (MMA, M=d_k N=64 K=64)
//   U^T = V^T T2^T   -> TMEM accumulator               (MMA, M=d_v N=64 K=64)
//   Vn^T = U^T - H^T W^T                                (MMA, B negated, K=d_k)
//   O1^T = H^T Q^T,  O2^T = Vn^T Aqk^T                 (MMAs)
//   o_r  = e^{G_r} scale O1[r] + O2[r]                 (state warps, bf16 out)
//   dH^T = (Vn diag-scaled by e^{G_C-G_r})^T K          (MMA, M=d_v N=d_k K=64)
//   H    <- e^{G_C} H + dH                             (state warps, f32 regs)
// The state is kept transposed (row j of H^T = column j of H) so that d_v is the
// MMA M dimension (128 TMEM lanes) everywhere; thread j of the state warps owns
// row j of H^T in 128 f32 registers.  d_k = d_v = 64 runs the same code with
// the upper halves of every tile zero.
//
// A chunk shorter than 64 rows (sequence end) gets g = beta = 0 in its padded
// rows: those rows then contribute nothing to any product (exactly), and the
// rows TMA reads past the sequence end (the next sequence, or zero fill past
// the tensor) are never stored.
//
// Warp roles (320 threads): warps 0-3 state/chain, 4-7 prep, 8 TMA, 9 MMA.
// All waits are bounded (gdn_device.cuh); a timeout sets g_err_prefill.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "gdn_device.cuh"
#include "gdn_internal.h"

namespace gdn {

__device__ uint32_t g_err_prefill;

namespace pf {

constexpr int C = 64;            // chunk rows
constexpr int kThreads = 320;    // 10 warps
constexpr int kAS = 65;          // f32 row stride of the A / T scratch

// Shared-memory layout (bytes from a 1024-aligned base).
constexpr uint32_t KQ0 = 0;          // [2 boxes][K 64x128B | Q 64x128B], 32 KB
constexpr uint32_t KQ1 = 32768;      // second stage
constexpr uint32_t VT = 65536;       // [2 boxes][64 x 128B], 16 KB
constexpr uint32_t HT = 81920;       // H^T bf16, [2 boxes][128 x 128B], 32 KB
constexpr uint32_t WB = 114688;      // W^T bf16, [128 rows (d_k) x 128B], 16 KB
constexpr uint32_t T1B = 131072;     // T1 bf16 [64 x 128B], 8 KB
constexpr uint32_t T2B = 139264;     // T2 bf16, 8 KB
constexpr uint32_t AQK = 147456;     // Aqk bf16 [64 x 128B], 8 KB
constexpr uint32_t VN = 155648;      // Vn^T bf16 [128 x 128B], 16 KB
constexpr uint32_t VNS = 172032;     // scaled Vn^T bf16, 16 KB
constexpr uint32_t AF = 188416;      // A f32 [64][65]
constexpr uint32_t TF = AF + 64 * kAS * 4;  // T f32 [64][65]
constexpr uint32_t GATE = TF + 64 * kAS * 4;  // prep-only gate arrays (one buffer)
constexpr int kPrepGateFloats = 64 * 7;       // G, beta, E1, E2[4][64]
constexpr uint32_t RING = GATE + kPrepGateFloats * 4;  // gate factors the state warps read
constexpr int kRingFloats = 132;              // e^{G_r}, e^{G_C - G_r}, e^{G_C}, pad
constexpr int kRingDepth = 4;                 // chunks in flight between prep and state
constexpr uint32_t BARS = RING + kRingDepth * kRingFloats * 4;
constexpr int kNumBars = 17;
constexpr uint32_t MISC = BARS + kNumBars * 8;
constexpr uint32_t kSmemBytes = MISC + 32;
constexpr uint32_t kSmemAlloc = kSmemBytes + 1024;
static_assert(kSmemAlloc <= 232448, "shared memory budget");
// X scratch of the blocked inverse lives in the T1B/T2B region (written later).
constexpr uint32_t XS = T1B;

// Prep-only gate arrays (floats from GATE).
constexpr int G_G = 0;      // G_r
constexpr int G_BET = 64;   // beta_r
constexpr int G_E1 = 128;   // e^{G_r - G_{16 floor(r/16)}}
constexpr int G_E2 = 192;   // [4][64]: e^{G_{16 b} - G_s} for s < 16 b, else 0
// Ring entries (floats from RING + (c % kRingDepth) * kRingFloats).
constexpr int R_EG = 0;     // e^{G_r}
constexpr int R_ECG = 64;   // e^{G_C - G_r}
constexpr int R_DEC = 128;  // e^{G_C}

// Barrier indices.
enum {
  B_KQ_FULL0 = 0, B_KQ_FULL1, B_KQ_EMPTY0, B_KQ_EMPTY1, B_V_FULL, B_V_EMPTY,
  B_P1_FULL, B_T_READY, B_WU_FULL, B_W_READY, B_H_READY, B_VN_FULL, B_VN_READY,
  B_DH_FULL, B_O_FULL, B_DRAIN, B_PREP_SYNC
};

// TMEM columns.
constexpr uint32_t TM_P1 = 0, TM_W = 64, TM_U0 = 128, TM_O1 = 256, TM_O2 = 320, TM_DH = 384;

struct Params {
  const float* g;
  const float* beta;
  const int32_t* cu_seqlens;
  const float* h0;
  float* hT;
  uint16_t* o;
  int gb_stride, num_seqs, total_tokens, H_k, H_v, D;
  float scale;
};

// Barrier among the 128 prep threads built on an mbarrier, so that it is
// bounded like every other wait (a bar.sync could block forever if one thread
// left early after a timeout).
__device__ __forceinline__ bool wg_sync(uint64_t* bar, uint32_t& phase, volatile int* abort_flag,
                                        uint32_t* err) {
  mbar_arrive(bar);
  const bool ok = mbar_wait(bar, phase, abort_flag, err, 64u);
  phase ^= 1u;
  return ok;
}

// [begin, end) of sequence n, clamped to the packed tensor.
__device__ __forceinline__ void seq_range(const int32_t* cu, int n, int total, int& b, int& e) {
  b = min(max(cu[n], 0), total);
  e = min(max(cu[n + 1], b), total);
}

// Write 8*NCH bf16 values (16-byte chunks c0 .. c0+NCH-1 of a 128-byte row) into
// a 128B-swizzled tile at `row`.
template <int NCH>
__device__ __forceinline__ void st_chunks_bf16(uint32_t tile, uint32_t row, int c0, const float* x) {
#pragma unroll
  for (int c = 0; c < NCH; ++c) {
    st_shared_v4(tile + sw128_offset(row, (c0 + c) * 16), pack_bf16x2(x[8 * c + 0], x[8 * c + 1]),
                 pack_bf16x2(x[8 * c + 2], x[8 * c + 3]), pack_bf16x2(x[8 * c + 4], x[8 * c + 5]),
                 pack_bf16x2(x[8 * c + 6], x[8 * c + 7]));
  }
}
__device__ __forceinline__ void st_row64_bf16(uint32_t tile, uint32_t row, const float* x) {
  st_chunks_bf16<8>(tile, row, 0, x);
}

}  // namespace pf

using namespace pf;

__global__ void __launch_bounds__(kThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + BARS);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + MISC + 4);
  float* Af = reinterpret_cast<float*>(smem + AF);
  float* Tf = reinterpret_cast<float*>(smem + TF);
  float* Xs = reinterpret_cast<float*>(smem + XS);

  const int warp = int(warp_id_sync());
  const int tid = threadIdx.x;
  const int D = p.D;
  const int nbox = D / 64;  // 64-column boxes per d_k / d_v row
  const int num_units = p.num_seqs * p.H_v;

  // Zero all shared memory once (the upper halves of d = 64 tiles stay zero).
  for (uint32_t i = tid * 16; i < kSmemBytes; i += kThreads * 16)
    *reinterpret_cast<uint4*>(smem + i) = make_uint4(0, 0, 0, 0);
  __syncthreads();
  if (tid == 0) {
    for (int b = 0; b < kNumBars; ++b) {
      uint32_t cnt = 1;
      if (b == B_T_READY || b == B_W_READY || b == B_H_READY || b == B_VN_READY ||
          b == B_PREP_SYNC)
        cnt = 128;
      mbar_init(&bars[b], cnt);
    }
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  if (warp == 0) tmem_alloc(tmem_slot, 512);
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  uint32_t* err = &g_err_prefill;

  if (warp == 8) {
    // ------------------------------------------------------------ TMA warp
    if (elect_one()) {
      int c = 0;  // running chunk counter over all units of this CTA
      int issued_kq = 0, issued_v = 0;  // loads issued (for the drain on exit)
      bool ok = true;
      for (int u = blockIdx.x; u < num_units && ok; u += gridDim.x) {
        const int n = u / p.H_v, h = u % p.H_v;
        const int hk = h / (p.H_v / p.H_k);
        int t_begin, t_end;
        seq_range(p.cu_seqlens, n, p.total_tokens, t_begin, t_end);
        for (int t0 = t_begin; t0 < t_end && ok; t0 += C, ++c) {
          const int st = c & 1;
          ok = mbar_wait(&bars[B_KQ_EMPTY0 + st], ((c >> 1) & 1) ^ 1, abort_flag, err, 1u);
          if (!ok) break;
          uint64_t* fb = &bars[B_KQ_FULL0 + st];
          mbar_arrive_expect_tx(fb, uint32_t(nbox) * 2 * 8192);
          uint8_t* kq = smem + (st ? KQ1 : KQ0);
          for (int b = 0; b < nbox; ++b) {
            tma_load_3d(kq + b * 16384, &tm_k, fb, b * 64, hk, t0);
            tma_load_3d(kq + b * 16384 + 8192, &tm_q, fb, b * 64, hk, t0);
          }
          issued_kq = c + 1;
          ok = mbar_wait(&bars[B_V_EMPTY], (c & 1) ^ 1, abort_flag, err, 1u);
          if (!ok) break;
          mbar_arrive_expect_tx(&bars[B_V_FULL], uint32_t(nbox) * 8192);
          for (int b = 0; b < nbox; ++b)
            tma_load_3d(smem + VT + b * 8192, &tm_v, &bars[B_V_FULL], b * 64, h, t0);
          issued_v = c + 1;
        }
      }
      // Drain: wait (bounded) for the last loads of each barrier so no copy is
      // still landing in shared memory when the CTA exits.
      for (int cc = issued_kq - 2; cc < issued_kq; ++cc)
        if (cc >= 0) mbar_wait(&bars[B_KQ_FULL0 + (cc & 1)], (cc >> 1) & 1, nullptr, err, 32u);
      if (issued_v > 0) mbar_wait(&bars[B_V_FULL], (issued_v - 1) & 1, nullptr, err, 32u);
    }
    __syncwarp();
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA warp
    if (elect_one()) {
      const uint32_t id_p1 = make_idesc_bf16(128, 64, 0, 0);
      const uint32_t id_wu = make_idesc_bf16(128, 64, 1, 0);
      const uint32_t id_vn = make_idesc_bf16(128, 64, 0, 1, /*b_neg=*/1);
      const uint32_t id_o1 = make_idesc_bf16(128, 64, 0, 0);
      const uint32_t id_dh = make_idesc_bf16(128, 128, 0, 1);
      const uint32_t id_o2 = make_idesc_bf16(128, 64, 0, 0);
      const int ksteps_d = D / 16;  // K steps over d_k
      int c = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < num_units && ok; u += gridDim.x) {
        const int n = u / p.H_v;
        int t_begin, t_end;
        seq_range(p.cu_seqlens, n, p.total_tokens, t_begin, t_end);
        for (int t0 = t_begin; t0 < t_end && ok; t0 += C, ++c) {
          const int st = c & 1;
          const uint32_t ph = c & 1;
          const uint32_t kq = sbase + (st ? KQ1 : KQ0);
          const uint32_t d_u = tmem + TM_U0 + 64u * uint32_t(st);
          // 1. P1 = [K;Q] K^T
          ok = mbar_wait(&bars[B_KQ_FULL0 + st], (c >> 1) & 1, abort_flag, err, 2u);
          if (!ok) break;
          tc_fence_after();
          for (int kk = 0; kk < ksteps_d; ++kk) {
            const uint32_t a = kq + (kk >> 2) * 16384 + (kk & 3) * 32;
            mma_bf16_ss(tmem + TM_P1, make_sdesc_sw128(a, 16, 1024), make_sdesc_sw128(a, 16, 1024),
                        id_p1, kk > 0);
          }
          mma_commit(&bars[B_P1_FULL]);
          // 2. W^T = K^T T1^T, U^T = V^T T2^T
          ok = mbar_wait(&bars[B_T_READY], ph, abort_flag, err, 2u) &&
               mbar_wait(&bars[B_V_FULL], ph, abort_flag, err, 2u);
          if (!ok) break;
          tc_fence_after();
          for (int kk = 0; kk < 4; ++kk) {
            mma_bf16_ss(tmem + TM_W, make_sdesc_sw128(kq + kk * 2048, 16384, 1024),
                        make_sdesc_sw128(sbase + T1B + kk * 32, 16, 1024), id_wu, kk > 0);
          }
          for (int kk = 0; kk < 4; ++kk) {
            mma_bf16_ss(d_u, make_sdesc_sw128(sbase + VT + kk * 2048, 8192, 1024),
                        make_sdesc_sw128(sbase + T2B + kk * 32, 16, 1024), id_wu, kk > 0);
          }
          mma_commit(&bars[B_V_EMPTY]);
          mma_commit(&bars[B_WU_FULL]);
          // 3. Vn^T = U^T - H^T W^T ; O1^T = H^T Q^T
          ok = mbar_wait(&bars[B_W_READY], ph, abort_flag, err, 2u) &&
               mbar_wait(&bars[B_H_READY], ph, abort_flag, err, 2u);
          if (!ok) break;
          tc_fence_after();
          for (int kk = 0; kk < ksteps_d; ++kk) {
            const uint32_t a = sbase + HT + (kk >> 2) * 16384 + (kk & 3) * 32;
            mma_bf16_ss(d_u, make_sdesc_sw128(a, 16, 1024),
                        make_sdesc_sw128(sbase + WB + kk * 2048, 8192, 1024), id_vn, 1);
          }
          mma_commit(&bars[B_VN_FULL]);
          for (int kk = 0; kk < ksteps_d; ++kk) {
            const uint32_t a = sbase + HT + (kk >> 2) * 16384 + (kk & 3) * 32;
            const uint32_t b = kq + (kk >> 2) * 16384 + 8192 + (kk & 3) * 32;
            mma_bf16_ss(tmem + TM_O1, make_sdesc_sw128(a, 16, 1024), make_sdesc_sw128(b, 16, 1024),
                        id_o1, kk > 0);
          }
          // 4. dH^T = Vns^T K ; O2^T = Vn^T Aqk^T
          ok = mbar_wait(&bars[B_VN_READY], ph, abort_flag, err, 2u);
          if (!ok) break;
          tc_fence_after();
          for (int kk = 0; kk < 4; ++kk) {
            mma_bf16_ss(tmem + TM_DH, make_sdesc_sw128(sbase + VNS + kk * 32, 16, 1024),
                        make_sdesc_sw128(kq + kk * 2048, 16384, 1024), id_dh, kk > 0);
          }
          mma_commit(&bars[B_DH_FULL]);
          for (int kk = 0; kk < 4; ++kk) {
            mma_bf16_ss(tmem + TM_O2, make_sdesc_sw128(sbase + VN + kk * 32, 16, 1024),
                        make_sdesc_sw128(sbase + AQK + kk * 32, 16, 1024), id_o2, kk > 0);
          }
          mma_commit(&bars[B_O_FULL]);
          mma_commit(&bars[B_KQ_EMPTY0 + st]);
        }
      }
      mma_commit(&bars[B_DRAIN]);
      mbar_wait(&bars[B_DRAIN], 0, nullptr, err, 8u);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------ prep warps
    const int pt = tid - 128;  // 0..127 == TMEM lane
    const uint32_t lane_off = uint32_t((warp & 3) * 32) << 16;
    uint32_t sync_phase = 0;
    uint64_t* psync = &bars[B_PREP_SYNC];
#define PREP_SYNC()                                          \
  if (!wg_sync(psync, sync_phase, abort_flag, err)) {        \
    ok = false;                                              \
    break;                                                   \
  }
    int c = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < num_units && ok; u += gridDim.x) {
      const int n = u / p.H_v, h = u % p.H_v;
      int t_begin, t_end;
        seq_range(p.cu_seqlens, n, p.total_tokens, t_begin, t_end);
      for (int t0 = t_begin; t0 < t_end && ok; t0 += C, ++c) {
        const int L = min(C, t_end - t0);
        const uint32_t ph = c & 1;
        float* gb = reinterpret_cast<float*>(smem + GATE);
        float* rb = reinterpret_cast<float*>(smem + RING) + (c % kRingDepth) * kRingFloats;
        // gates of this chunk (padded rows: g = beta = 0)
        if (pt < 64) {
          const bool valid = pt < L;
          gb[G_G + pt] = valid ? p.g[size_t(t0 + pt) * p.gb_stride + h] : 0.f;
          gb[G_BET + pt] = valid ? p.beta[size_t(t0 + pt) * p.gb_stride + h] : 0.f;
        }
        PREP_SYNC();
        if (pt < 32) {  // inclusive scan of g over 64 rows (2 per lane)
          float a0 = gb[G_G + 2 * pt], a1 = gb[G_G + 2 * pt + 1];
          float s = a0 + a1;
#pragma unroll
          for (int off = 1; off < 32; off <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, s, off);
            if (pt >= off) s += y;
          }
          const float excl = s - (a0 + a1);
          gb[G_G + 2 * pt] = excl + a0;
          gb[G_G + 2 * pt + 1] = excl + a0 + a1;
        }
        PREP_SYNC();
        {
          const float GC = gb[G_G + 63];
          if (pt < 64) {
            const float Gr = gb[G_G + pt];
            rb[R_EG + pt] = __expf(Gr);
            rb[R_ECG + pt] = __expf(GC - Gr);
            gb[G_E1 + pt] = __expf(Gr - gb[G_G + (pt & ~15)]);
          }
          for (int e = pt; e < 256; e += 128) {  // E2[b][s] = e^{G_{16b} - G_s}, s < 16b
            const int bb = e >> 6, s = e & 63;
            gb[G_E2 + e] = (s < 16 * bb) ? __expf(gb[G_G + 16 * bb] - gb[G_G + s]) : 0.f;
          }
          if (pt == 0) rb[R_DEC] = __expf(GC);
        }
        PREP_SYNC();
        // P1 row pt: K K^T (pt < 64) or Q K^T (pt >= 64)
        ok = mbar_wait(&bars[B_P1_FULL], ph, abort_flag, err, 4u);
        if (!ok) break;
        tc_fence_after();
        {
          float row[64];
          float tmp[32];
          tmem_ld32(tmem + lane_off + TM_P1, tmp);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) row[i] = tmp[i];
          tmem_ld32(tmem + lane_off + TM_P1 + 32, tmp);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) row[32 + i] = tmp[i];
          const int r = pt & 63;
          // row[s] *= Gamma[r][s] = e^{G_r - G_s} (s <= r), as a product of two factors
          // <= 1 for blocks of s before r's 16-row block (E1 * E2), directly inside it.
          const int rb = r >> 4;
          const float Gr = gb[G_G + r];
          const float e1 = gb[G_E1 + r];
          const float* e2 = gb + G_E2 + 64 * rb;
#pragma unroll
          for (int sb = 0; sb < 4; ++sb) {
            if (sb < rb) {
#pragma unroll
              for (int jj = 0; jj < 16; ++jj) row[16 * sb + jj] *= e1 * e2[16 * sb + jj];
            } else if (sb == rb) {
#pragma unroll
              for (int jj = 0; jj < 16; ++jj) {
                const int s = 16 * sb + jj;
                row[s] = (s <= r) ? row[s] * __expf(Gr - gb[G_G + s]) : 0.f;
              }
            } else {
#pragma unroll
              for (int jj = 0; jj < 16; ++jj) row[16 * sb + jj] = 0.f;
            }
          }
          if (pt < 64) {
            const float br = gb[G_BET + r];
#pragma unroll
            for (int s = 0; s < 64; ++s) Af[r * kAS + s] = (s < r) ? br * row[s] : 0.f;
          } else {
            const float sc = p.scale;
#pragma unroll
            for (int s = 0; s < 64; ++s) row[s] *= sc;
            st_row64_bf16(sbase + AQK, uint32_t(r), row);
          }
        }
        tc_fence_before();
        PREP_SYNC();
        // T = (I + A)^{-1}: 16x16 diagonal blocks by forward substitution ...
        if (pt < 64) {
          const int d = pt >> 4, j = pt & 15;
          float x[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) x[i] = (i == j) ? 1.f : 0.f;
#pragma unroll
          for (int i = 1; i < 16; ++i) {
            float s = 0.f;
#pragma unroll
            for (int l = 0; l < i; ++l) s = fmaf(Af[(16 * d + i) * kAS + 16 * d + l], x[l], s);
            if (i > j) x[i] = -s;
          }
#pragma unroll
          for (int i = 0; i < 16; ++i) Tf[(16 * d + i) * kAS + 16 * d + j] = x[i];
        }
        PREP_SYNC();
        // ... then the off-diagonal blocks by block diagonals L = 1, 2, 3:
        //   X = sum_{l in blocks bj..bi-1} A_{bi,l} T_{l,bj};  T_{bi,bj} = -T_{bi,bi} X
        for (int Ld = 1; Ld < 4; ++Ld) {
          const int ntask = (4 - Ld) * 256;
          for (int t = pt; t < ntask; t += 128) {
            const int blk = t >> 8, e = t & 255, i = e >> 4, jj = e & 15;
            const int bi = Ld + blk, bj = blk;
            float s = 0.f;
            const float* arow = Af + (16 * bi + i) * kAS;
            for (int l = 16 * bj; l < 16 * bi; ++l) s = fmaf(arow[l], Tf[l * kAS + 16 * bj + jj], s);
            Xs[t] = s;
          }
          PREP_SYNC();
          for (int t = pt; t < ntask; t += 128) {
            const int blk = t >> 8, e = t & 255, i = e >> 4, jj = e & 15;
            const int bi = Ld + blk, bj = blk;
            const float* trow = Tf + (16 * bi + i) * kAS + 16 * bi;
            float s = 0.f;
#pragma unroll
            for (int l = 0; l < 16; ++l) s = fmaf(trow[l], Xs[blk * 256 + l * 16 + jj], s);
            Tf[(16 * bi + i) * kAS + 16 * bj + jj] = -s;
          }
          PREP_SYNC();
        }
        if (!ok) break;
        // T1 = T diag(beta e^G) (rows pt < 64), T2 = T diag(beta) (rows pt >= 64)
        {
          const int r = pt & 63;
          float row[64];
#pragma unroll
          for (int s = 0; s < 64; ++s) {
            const float sc = (pt < 64) ? gb[G_BET + s] * rb[R_EG + s] : gb[G_BET + s];
            row[s] = (s <= r) ? Tf[r * kAS + s] * sc : 0.f;
          }
          st_row64_bf16(sbase + (pt < 64 ? T1B : T2B), uint32_t(r), row);
        }
        fence_proxy_async_smem();
        mbar_arrive(&bars[B_T_READY]);
        // W^T row pt (d_k index) -> bf16 -> WB (MN-major B of the chain MMA)
        ok = mbar_wait(&bars[B_WU_FULL], ph, abort_flag, err, 4u);
        if (!ok) break;
        tc_fence_after();
        {
          float row[64];
          float tmp[32];
          tmem_ld32(tmem + lane_off + TM_W, tmp);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) row[i] = tmp[i];
          tmem_ld32(tmem + lane_off + TM_W + 32, tmp);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) row[32 + i] = tmp[i];
          st_row64_bf16(sbase + WB, uint32_t(pt), row);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&bars[B_W_READY]);
      }
    }
#undef PREP_SYNC
  } else {
    // ------------------------------------------------------------ state warps
    const int j = tid;  // v index == TMEM lane == row of H^T
    const uint32_t lane_off = uint32_t(warp * 32) << 16;
    const bool jv = j < D;
    int c = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < num_units && ok; u += gridDim.x) {
      const int n = u / p.H_v, h = u % p.H_v;
      int t_begin, t_end;
        seq_range(p.cu_seqlens, n, p.total_tokens, t_begin, t_end);
      const size_t state_off = (size_t(n) * p.H_v + h) * size_t(D) * D;
      float H[128];
#pragma unroll
      for (int i = 0; i < 128; ++i) H[i] = 0.f;
      if (p.h0 != nullptr && jv) {
#pragma unroll
        for (int i = 0; i < 128; ++i)
          if (i < D) H[i] = p.h0[state_off + size_t(i) * D + j];
      }
      for (int t0 = t_begin; t0 < t_end && ok; t0 += C, ++c) {
        const int L = min(C, t_end - t0);
        const uint32_t ph = c & 1;
        const float* rb =
            reinterpret_cast<const float*>(smem + RING) + (c % kRingDepth) * kRingFloats;
        // (a) H^T row j -> bf16 -> HT (K-major A operand)
#pragma unroll
        for (int b = 0; b < 2; ++b) st_row64_bf16(sbase + HT + b * 16384, uint32_t(j), H + 64 * b);
        fence_proxy_async_smem();
        mbar_arrive(&bars[B_H_READY]);
        // (b) Vn^T row j -> bf16 (plain and scaled by e^{G_C - G_r})
        ok = mbar_wait(&bars[B_VN_FULL], ph, abort_flag, err, 16u);
        if (!ok) break;
        tc_fence_after();
        {
          const uint32_t d_u = tmem + lane_off + TM_U0 + 64u * uint32_t(c & 1);
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            float vn[32];
            tmem_ld32(d_u + 32u * half, vn);
            tmem_ld_wait();
            st_chunks_bf16<4>(sbase + VN, uint32_t(j), 4 * half, vn);
#pragma unroll
            for (int r = 0; r < 32; ++r) vn[r] *= rb[R_ECG + 32 * half + r];
            st_chunks_bf16<4>(sbase + VNS, uint32_t(j), 4 * half, vn);
          }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&bars[B_VN_READY]);
        // (c) H <- e^{G_C} H + dH
        ok = mbar_wait(&bars[B_DH_FULL], ph, abort_flag, err, 16u);
        if (!ok) break;
        tc_fence_after();
        {
          const float dec = rb[R_DEC];
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            float tmp[32];
            tmem_ld32(tmem + lane_off + TM_DH + 32u * q4, tmp);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i) H[32 * q4 + i] = fmaf(dec, H[32 * q4 + i], tmp[i]);
          }
        }
        // (d) o_r = e^{G_r} scale O1[r] + O2[r]
        ok = mbar_wait(&bars[B_O_FULL], ph, abort_flag, err, 16u);
        if (!ok) break;
        tc_fence_after();
        {
          const float sc = p.scale;
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            float o1[16], o2[16];
            tmem_ld16(tmem + lane_off + TM_O1 + 16u * q4, o1);
            tmem_ld16(tmem + lane_off + TM_O2 + 16u * q4, o2);
            tmem_ld_wait();
            if (jv) {
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                const int r = 16 * q4 + i;
                if (r < L) {
                  const float val = fmaf(rb[R_EG + r] * sc, o1[i], o2[i]);
                  p.o[(size_t(t0 + r) * p.H_v + h) * D + j] =
                      __bfloat16_as_ushort(__float2bfloat16_rn(val));
                }
              }
            }
          }
        }
        tc_fence_before();
      }
      if (ok && p.hT != nullptr && jv) {
#pragma unroll
        for (int i = 0; i < 128; ++i)
          if (i < D) p.hT[state_off + size_t(i) * D + j] = H[i];
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

size_t prefill_workspace_bytes(int, int, int, int, int) { return 0; }

cudaError_t launch_prefill(const uint16_t* q, const uint16_t* k, int qk_stride,
                           const uint16_t* v, int v_stride, const float* g, const float* beta,
                           int gb_stride, const int32_t* cu_seqlens, int num_seqs,
                           int total_tokens, const float* h0, float* hT, uint16_t* o, int H_k,
                           int H_v, int D, float scale, void* workspace, cudaStream_t s) {
  (void)workspace;
  CUtensorMap tq, tk, tv;
  {
    uint64_t dims[3] = {uint64_t(D), uint64_t(H_k), uint64_t(total_tokens)};
    uint64_t strides[2] = {uint64_t(D) * 2, uint64_t(qk_stride) * 2};
    uint32_t box[3] = {64, 1, 64};
    if (!encode_tmap_bf16(&tq, q, 3, dims, strides, box, true)) return cudaErrorInvalidValue;
    if (!encode_tmap_bf16(&tk, k, 3, dims, strides, box, true)) return cudaErrorInvalidValue;
  }
  {
    uint64_t dims[3] = {uint64_t(D), uint64_t(H_v), uint64_t(total_tokens)};
    uint64_t strides[2] = {uint64_t(D) * 2, uint64_t(v_stride) * 2};
    uint32_t box[3] = {64, 1, 64};
    if (!encode_tmap_bf16(&tv, v, 3, dims, strides, box, true)) return cudaErrorInvalidValue;
  }
  Params p;
  p.g = g;
  p.beta = beta;
  p.cu_seqlens = cu_seqlens;
  p.h0 = h0;
  p.hT = hT;
  p.o = o;
  p.gb_stride = gb_stride;
  p.num_seqs = num_seqs;
  p.total_tokens = total_tokens;
  p.H_k = H_k;
  p.H_v = H_v;
  p.D = D;
  p.scale = scale;
  cudaError_t e = cudaFuncSetAttribute(prefill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       int(kSmemAlloc));
  if (e != cudaSuccess) return e;
  const int units = num_seqs * H_v;
  int grid = units < sm_count() ? units : sm_count();
  prefill_kernel<<<grid, kThreads, kSmemAlloc, s>>>(tq, tk, tv, p);
  return cudaGetLastError();
}

// Read and clear this file's device error word (host; synchronous).
cudaError_t take_err_prefill(uint32_t* out) {
  uint32_t zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(out, g_err_prefill, sizeof(uint32_t));
  if (e != cudaSuccess) return e;
  return cudaMemcpyToSymbol(g_err_prefill, &zero, sizeof(uint32_t));
}

}  // namespace gdn
