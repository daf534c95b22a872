// gdn_prefill.cu -- chunk-parallel gated delta rule prefill on sm_100a.
//
// Page "ssm_gdn_tc_route.rs" names the piece this kernel replaces: the prefill
// "state spine" (chunk_delta_h) that carries the f32 recurrent state across
// chunks with bf16 tensor-core operands and an f32 accumulator.  Here the whole
// chunk step is one kernel, and each (sequence, v-head) unit is handled by a
// cluster of three CTAs on three SMs:
//
//   rank 0, the SPINE: holds H (f32, registers) and runs the per-chunk critical
//     chain  Vn^T = U^T - H^T W^T,  dH^T = (e^{G_C - G_r} Vn)^T K,
//     H <- e^{G_C} H + dH,  and the outputs  o_r = e^{G_r} scale (Q H)_r +
//     (Aqk Vn)_r  (tcgen05 MMAs, TMEM accumulators, M = d_v = 128 lanes);
//   ranks 1 and 2, the PREPS: compute everything that does not depend on H for
//     alternate chunks (rank 1 even chunks, rank 2 odd ones), two chunks at a
//     time per CTA (one per 4-warp group):
//       P1 = [K;Q] K^T                                 (MMA)
//       A[r][s]   = beta_r e^{G_r-G_s} k_r.k_s, s < r   (f32)
//       Aqk[r][s] = scale e^{G_r-G_s} q_r.k_s, s <= r
//       T = (I + A)^{-1}                               (blocked, f32, CUDA cores)
//       W^T = K^T (T diag(beta e^G))^T,  U^T = V^T (T diag(beta))^T   (MMAs)
//     and store W^T, U^T, Aqk (bf16) and the gate factors straight into one of
//     the spine's two shared-memory slots (distributed shared memory stores,
//     then a remote mbarrier arrive).  The spine frees a slot the same way.
//
// This is the WY/UT chunk form: within a chunk of rows r = 0..L-1 with
// G_r = g_0 + ... + g_r, (I + A) Vn = diag(beta) V - diag(beta e^G) K H, the
// outputs and the next state follow; the result equals the token recurrence up
// to rounding.  A chunk shorter than 64 rows gets g = beta = 0 in its padded
// rows, which then contribute nothing (exactly); padded rows are never stored.
// d_k = d_v = 64 runs the same code with the upper halves of every tile zero.
//
// No TMA multicast: every CTA loads its own K/Q/V tiles (L2 serves re-reads).
// Every wait is bounded (gdn_device.cuh); a timeout sets g_err_prefill and the
// kernel returns instead of hanging.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "gdn_device.cuh"
#include "gdn_internal.h"

namespace gdn {

__device__ uint32_t g_err_prefill;

namespace pf {

constexpr int C = 64;          // chunk rows
constexpr int kThreads = 320;  // 10 warps
constexpr int kCluster = 3;    // spine + 2 preps
constexpr int kAS = 68;        // f32 row stride of the A / T scratch (16-byte rows)

// ---- spine shared memory (bytes from a 1024-aligned base)
constexpr uint32_t S_KQ = 0;            // [2 stages][2 boxes][K 64x128B | Q 64x128B]
constexpr uint32_t S_HT = 65536;        // H^T bf16, [2 boxes][128 x 128B]
constexpr uint32_t S_VN = 98304;        // Vn^T bf16 [128 x 128B]
constexpr uint32_t S_VNS = 114688;      // scaled Vn^T bf16
constexpr uint32_t S_OST = 131072;      // output staging [64 rows][d_v] bf16, row-major
constexpr uint32_t S_SLOT = 147456;     // 2 slots of {W^T, U^T, Aqk}
constexpr uint32_t SL_W = 0;            // W^T bf16 [128 (d_k) x 128B] (MN-major B operand)
constexpr uint32_t SL_U = 16384;        // U^T bf16 [128 (d_v) x 128B] (swizzled rows)
constexpr uint32_t SL_AQK = 32768;      // Aqk bf16 [64 x 128B] (K-major B operand)
constexpr uint32_t SL_BYTES = 40960;
constexpr uint32_t S_SGATE = S_SLOT + 2 * SL_BYTES;  // 2 x [e^{G_r} 64 | e^{G_C-G_r} 64 | e^{G_C}]
constexpr uint32_t SG_FLOATS = 132;
constexpr uint32_t S_BARS = S_SGATE + 2 * SG_FLOATS * 4;
// ---- prep shared memory: two item groups of P_WG bytes
constexpr uint32_t P_KQ = 0;        // [2 boxes][K | Q]
constexpr uint32_t P_V = 32768;     // [2 boxes][64 x 128B]
constexpr uint32_t P_T1B = 49152;   // T diag(beta e^G) bf16 [64 x 128B]
constexpr uint32_t P_T2B = 57344;   // T diag(beta) bf16
constexpr uint32_t P_AF = 65536;    // A f32 [64][kAS]
constexpr uint32_t P_TF = P_AF + 64 * kAS * 4;  // T f32 [64][kAS]
constexpr uint32_t P_XS = P_TF + 64 * kAS * 4;  // block-product scratch, 3 x 16 x 16 f32
constexpr uint32_t P_GATE = P_XS + 3 * 256 * 4;
constexpr int PG_G = 0, PG_BET = 64, PG_E1 = 128, PG_E2 = 192, PG_BEG = 448, PG_EG = 512,
              PG_ECG = 576, PG_DEC = 640;  // floats
constexpr uint32_t P_AQK = (P_GATE + 644 * 4 + 1023) / 1024 * 1024;  // Aqk bf16 [64][128B] staging
constexpr uint32_t P_WG = P_AQK + 8192;
constexpr uint32_t P_BARS = 2 * P_WG;
constexpr uint32_t BAR_BYTES = 24 * 8;
constexpr uint32_t kSmemBytes =
    ((S_BARS > P_BARS ? S_BARS : P_BARS) + BAR_BYTES + 16 + 15) / 16 * 16;
constexpr uint32_t kSmemAlloc = kSmemBytes + 1024;
static_assert(kSmemAlloc <= 232448, "shared memory budget");
static_assert(S_BARS % 8 == 0 && P_BARS % 8 == 0, "barrier alignment");

// ---- barriers (spine)
enum {
  SB_KQF = 0,     // +stage: K/Q tiles landed (TMA)
  SB_KQE = 2,     // +stage: K/Q tiles free (MMA commit)
  SB_SLOTF = 4,   // +slot: a prep filled the slot (128 remote arrivals)
  SB_HREADY = 6,  // H^T bf16 written (128)
  SB_VNFULL = 7,  // -H^T W^T done (commit)
  SB_VNREADY = 8, // Vn / scaled Vn written (128)
  SB_DHFULL = 9,  // H += dH done (commit)
  SB_OFULL = 10,  // +buf: O1, O2 done (commit)
  SB_OFREE = 12,  // +buf: O1, O2 read back (128)
  SB_EPISYNC = 14,
  SB_DRAIN = 15,
  SB_EXIT = 16,
  SB_COUNT = 17
};
// ---- barriers (prep); per group w: base + w
enum {
  PB_KQVF = 0, PB_KQVE = 2, PB_P1F = 4, PB_P1FREE = 6, PB_TREADY = 8, PB_WUF = 10, PB_SYNC = 12,
  // +group: the spine released this CTA's slot for the group that writes it
  // next (slot item ks is followed by ks + 1, which group (ks + 1) & 1 writes);
  // 128 remote arrivals each
  PB_SLOTFREE = 14,
  PB_DRAIN = 16,
  PB_EXIT = 17,
  PB_COUNT = 18
};

// ---- TMEM columns
// spine: Vn, O1 x2, O2 x2, and the state H^T itself (f32, lane j = row j)
constexpr uint32_t ST_VN = 0, ST_O1 = 64, ST_O2 = 192, ST_H = 320;
constexpr uint32_t PT_P1 = 0, PT_W = 64, PT_U = 128, PT_WG = 192;    // prep, per group

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

// Walks the chunks of the units this cluster owns (u = cluster, += clusters);
// `c` counts chunks over all of them and is the same in every role.
struct ChunkIter {
  int u, n, h, t0, tb, te, c;
  bool ok;
};

__device__ __forceinline__ void seq_range(const Params& p, int n, int& b, int& e) {
  b = min(max(p.cu_seqlens[n], 0), p.total_tokens);
  e = min(max(p.cu_seqlens[n + 1], b), p.total_tokens);
}

__device__ __forceinline__ void it_load_unit(ChunkIter& it, const Params& p) {
  it.n = it.u / p.H_v;
  it.h = it.u % p.H_v;
  seq_range(p, it.n, it.tb, it.te);
  it.t0 = it.tb;
}

__device__ __forceinline__ void it_skip_empty(ChunkIter& it, const Params& p, int ustep) {
  const int units = p.num_seqs * p.H_v;
  while (it.ok && it.t0 >= it.te) {
    it.u += ustep;
    if (it.u >= units) {
      it.ok = false;
      break;
    }
    it_load_unit(it, p);
  }
}

__device__ __forceinline__ void it_start(ChunkIter& it, const Params& p, int u0, int ustep) {
  it.u = u0;
  it.c = 0;
  it.ok = u0 < p.num_seqs * p.H_v;
  if (it.ok) it_load_unit(it, p);
  it_skip_empty(it, p, ustep);
}

__device__ __forceinline__ void it_next(ChunkIter& it, const Params& p, int ustep) {
  it.t0 += C;
  ++it.c;
  it_skip_empty(it, p, ustep);
}

// Advance to the first chunk at or after the current one with c % 4 == sel.
__device__ __forceinline__ void it_align(ChunkIter& it, const Params& p, int ustep, int sel) {
  while (it.ok && (it.c & 3) != sel) it_next(it, p, ustep);
}

// Bounded barrier among the 128 threads of one warpgroup (mbarrier based).
struct WgSync {
  uint64_t* bar;
  uint32_t phase;
  __device__ __forceinline__ bool operator()(volatile int* abort, uint32_t* err) {
    mbar_arrive(bar);
    const bool ok = mbar_wait(bar, phase, abort, err, 64u);
    phase ^= 1u;
    return ok;
  }
};

template <int NCH>
__device__ __forceinline__ void pack_chunks(const float* x, uint32_t* out) {
#pragma unroll
  for (int c = 0; c < 4 * NCH; ++c) out[c] = pack_bf16x2(x[2 * c], x[2 * c + 1]);
}

// Write 64 bf16 values as a 128-byte row of a 128B-swizzled tile (local smem).
__device__ __forceinline__ void st_row64_bf16(uint32_t tile, uint32_t row, const float* x) {
#pragma unroll
  for (int c = 0; c < 8; ++c)
    st_shared_v4(tile + sw128_offset(row, c * 16), pack_bf16x2(x[8 * c + 0], x[8 * c + 1]),
                 pack_bf16x2(x[8 * c + 2], x[8 * c + 3]), pack_bf16x2(x[8 * c + 4], x[8 * c + 5]),
                 pack_bf16x2(x[8 * c + 6], x[8 * c + 7]));
}

// Same, from 32 packed words, into another CTA's shared memory.
__device__ __forceinline__ void st_row64_remote(uint32_t tile_cluster, uint32_t row,
                                                const uint32_t* w) {
#pragma unroll
  for (int c = 0; c < 8; ++c)
    st_cluster_v4(tile_cluster + sw128_offset(row, c * 16), w[4 * c], w[4 * c + 1], w[4 * c + 2],
                  w[4 * c + 3]);
}

// Read 64 bf16 of a swizzled row back as f32.
__device__ __forceinline__ void ld_row64_bf16(const uint8_t* tile, uint32_t row, float* x) {
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    const uint4 v = *reinterpret_cast<const uint4*>(tile + sw128_offset(row, c * 16));
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      x[8 * c + 2 * k] = __uint_as_float(w[k] << 16);
      x[8 * c + 2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
    }
  }
}

__device__ __forceinline__ void tmem_ld64(uint32_t taddr, float* x) {
  float a[32], b[32];
  tmem_ld32(taddr, a);
  tmem_ld32(taddr + 32, b);
  tmem_ld_wait();
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    x[i] = a[i];
    x[32 + i] = b[i];
  }
}

// ---------------------------------------------------------------------------
// T = (I + A)^{-1} for a strictly lower triangular 64x64 A (f32, row stride
// kAS), by 16x16 blocks: the diagonal blocks by forward substitution, then the
// block diagonals L = 1, 2, 3:
//   X = sum_{l in blocks bj .. bi-1} A_{bi,l} T_{l,bj};   T_{bi,bj} = -T_{bi,bi} X
// 128 threads; every phase is a set of independent 2-column tasks.
// ---------------------------------------------------------------------------
template <int LD>
__device__ __forceinline__ void level_x(const float* Af, const float* Tf, float* Xs, int p) {
  constexpr int NB = 4 - LD;
  constexpr int PARTS = (LD == 3) ? 3 : 1;
  constexpr int KLEN = 16 * LD / PARTS;
  constexpr int NT = NB * PARTS;  // tasks per thread (128 tasks per block-part)
  const int i = p >> 3, q = p & 7;
  float acc[NT][2];
#pragma unroll
  for (int t = 0; t < NT; ++t) acc[t][0] = acc[t][1] = 0.f;
#pragma unroll
  for (int l = 0; l < KLEN; l += 4) {
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      const int b = t / PARTS, part = t % PARTS;
      const int bi = b + LD, bj = b, k0 = 16 * bj + part * KLEN;
      const float4 a = *reinterpret_cast<const float4*>(Af + (16 * bi + i) * kAS + k0 + l);
      const float* tc = Tf + (k0 + l) * kAS + 16 * bj + 2 * q;
      const float2 t0 = *reinterpret_cast<const float2*>(tc);
      const float2 t1 = *reinterpret_cast<const float2*>(tc + kAS);
      const float2 t2 = *reinterpret_cast<const float2*>(tc + 2 * kAS);
      const float2 t3 = *reinterpret_cast<const float2*>(tc + 3 * kAS);
      acc[t][0] = fmaf(a.x, t0.x, acc[t][0]);
      acc[t][1] = fmaf(a.x, t0.y, acc[t][1]);
      acc[t][0] = fmaf(a.y, t1.x, acc[t][0]);
      acc[t][1] = fmaf(a.y, t1.y, acc[t][1]);
      acc[t][0] = fmaf(a.z, t2.x, acc[t][0]);
      acc[t][1] = fmaf(a.z, t2.y, acc[t][1]);
      acc[t][0] = fmaf(a.w, t3.x, acc[t][0]);
      acc[t][1] = fmaf(a.w, t3.y, acc[t][1]);
    }
  }
#pragma unroll
  for (int t = 0; t < NT; ++t)
    *reinterpret_cast<float2*>(Xs + t * 256 + i * 16 + 2 * q) = make_float2(acc[t][0], acc[t][1]);
}

template <int LD>
__device__ __forceinline__ void level_t(float* Tf, const float* Xs, int p) {
  constexpr int NB = 4 - LD;
  constexpr int PARTS = (LD == 3) ? 3 : 1;
  const int i = p >> 3, q = p & 7;
#pragma unroll
  for (int b = 0; b < NB; ++b) {
    const int bi = b + LD, bj = b;
    const float* tr = Tf + (16 * bi + i) * kAS + 16 * bi;
    float y0 = 0.f, y1 = 0.f;
#pragma unroll
    for (int l = 0; l < 16; l += 4) {
      const float4 a = *reinterpret_cast<const float4*>(tr + l);
      const float av[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        float x0 = 0.f, x1 = 0.f;
#pragma unroll
        for (int part = 0; part < PARTS; ++part) {
          const float2 xv = *reinterpret_cast<const float2*>(Xs + (b * PARTS + part) * 256 +
                                                             (l + m) * 16 + 2 * q);
          x0 += xv.x;
          x1 += xv.y;
        }
        y0 = fmaf(av[m], x0, y0);
        y1 = fmaf(av[m], x1, y1);
      }
    }
    *reinterpret_cast<float2*>(Tf + (16 * bi + i) * kAS + 16 * bj + 2 * q) = make_float2(-y0, -y1);
  }
}

__device__ __forceinline__ bool invert_unit_lower64(const float* Af, float* Tf, float* Xs, int p,
                                                    WgSync& sync, volatile int* abort,
                                                    uint32_t* err) {
  const int lane = p & 31, d = p >> 5;
  if (lane < 16) {  // diagonal block d, column j
    const int j = lane;
    const float* Ab = Af + (16 * d) * kAS + 16 * d;
    float x[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) x[i] = (i == j) ? 1.f : 0.f;
#pragma unroll
    for (int i = 1; i < 16; ++i) {
      float s = 0.f;
#pragma unroll
      for (int l = 0; l < i; ++l) s = fmaf(Ab[i * kAS + l], x[l], s);
      if (i > j) x[i] = -s;
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) Tf[(16 * d + i) * kAS + 16 * d + j] = x[i];
  }
  if (!sync(abort, err)) return false;
  level_x<1>(Af, Tf, Xs, p);
  if (!sync(abort, err)) return false;
  level_t<1>(Tf, Xs, p);
  if (!sync(abort, err)) return false;
  level_x<2>(Af, Tf, Xs, p);
  if (!sync(abort, err)) return false;
  level_t<2>(Tf, Xs, p);
  if (!sync(abort, err)) return false;
  level_x<3>(Af, Tf, Xs, p);
  if (!sync(abort, err)) return false;
  level_t<3>(Tf, Xs, p);
  return sync(abort, err);
}

}  // namespace pf

using namespace pf;

__global__ void __cluster_dims__(kCluster, 1, 1) __launch_bounds__(kThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t rank = cluster_ctarank();
  const bool spine = rank == 0;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (spine ? S_BARS : P_BARS));
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 24);  // after 24 barrier slots
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 24) + 1;
  uint32_t* err = &g_err_prefill;

  const int warp = int(warp_id_sync());
  const int tid = threadIdx.x;
  const int D = p.D;
  const int nbox = D / 64;
  const int u0 = int(cluster_id_x());
  const int ustep = int(num_clusters_x());

  for (uint32_t i = tid * 16; i < kSmemBytes; i += kThreads * 16)
    *reinterpret_cast<uint4*>(smem + i) = make_uint4(0, 0, 0, 0);
  __syncthreads();
  if (tid == 0) {
    if (spine) {
      for (int b = 0; b < SB_COUNT; ++b) {
        uint32_t cnt = 1;
        if (b == SB_SLOTF || b == SB_SLOTF + 1 || b == SB_HREADY || b == SB_VNREADY ||
            b == SB_OFREE || b == SB_OFREE + 1 || b == SB_EPISYNC)
          cnt = 128;
        if (b == SB_EXIT) cnt = kCluster;
        mbar_init(&bars[b], cnt);
      }
    } else {
      for (int b = 0; b < PB_COUNT; ++b) {
        uint32_t cnt = 1;
        if (b == PB_P1FREE || b == PB_P1FREE + 1 || b == PB_TREADY || b == PB_TREADY + 1 ||
            b == PB_SYNC || b == PB_SYNC + 1 || b == PB_SLOTFREE || b == PB_SLOTFREE + 1)
          cnt = 128;
        if (b == PB_EXIT) cnt = kCluster;
        mbar_init(&bars[b], cnt);
      }
    }
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  if (warp == 0) tmem_alloc(tmem_slot, 512);
  __syncthreads();
  cluster_sync_start();  // every CTA's barriers are initialised before any remote arrive
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int ksteps_d = D / 16;

  if (spine) {
    // =====================================================================
    // SPINE
    // =====================================================================
    if (warp == 8) {
      // ---------------- TMA: K and Q tiles of every chunk (2 stages)
      if (elect_one()) {
        ChunkIter it;
        it_start(it, p, u0, ustep);
        int issued = 0;
        while (it.ok) {
          const int c = it.c, st = c & 1;
          if (!mbar_wait(&bars[SB_KQE + st], ((c >> 1) & 1) ^ 1, abort_flag, err, 1u)) break;
          uint64_t* fb = &bars[SB_KQF + st];
          mbar_arrive_expect_tx(fb, uint32_t(nbox) * 2 * 8192);
          uint8_t* kq = smem + S_KQ + st * 32768;
          const int hk = it.h / (p.H_v / p.H_k);
          for (int b = 0; b < nbox; ++b) {
            tma_load_3d(kq + b * 16384, &tm_k, fb, b * 64, hk, it.t0);
            tma_load_3d(kq + b * 16384 + 8192, &tm_q, fb, b * 64, hk, it.t0);
          }
          issued = c + 1;
          it_next(it, p, ustep);
        }
        for (int cc = issued - 2; cc < issued; ++cc)
          if (cc >= 0) mbar_wait(&bars[SB_KQF + (cc & 1)], (cc >> 1) & 1, nullptr, err, 32u);
      }
      __syncwarp();
    } else if (warp == 9) {
      // ---------------- MMA issue (one thread), chunk by chunk
      if (elect_one()) {
        const uint32_t id_vn = make_idesc_bf16(128, 64, 0, 1, /*b_neg=*/1);
        const uint32_t id_o1 = make_idesc_bf16(128, 64, 0, 0);
        const uint32_t id_dh = make_idesc_bf16(128, 128, 0, 1);
        const uint32_t id_o2 = make_idesc_bf16(128, 64, 0, 0);
        ChunkIter it;
        it_start(it, p, u0, ustep);
        while (it.ok) {
          const int c = it.c, st = c & 1, ob = c & 1;
          const uint32_t kq = sbase + S_KQ + st * 32768;
          const uint32_t slot = sbase + S_SLOT + st * SL_BYTES;
          if (!mbar_wait(&bars[SB_KQF + st], (c >> 1) & 1, abort_flag, err, 2u)) break;
          if (!mbar_wait_cluster(&bars[SB_SLOTF + st], (c >> 1) & 1, abort_flag, err, 2u)) break;
          if (!mbar_wait(&bars[SB_HREADY], c & 1, abort_flag, err, 2u)) break;
          fence_proxy_async_smem();
          tc_fence_after();
          // Vn^T := -H^T W^T   (U^T is added by the state warps)
          for (int kk = 0; kk < ksteps_d; ++kk) {
            const uint32_t a = sbase + S_HT + (kk >> 2) * 16384 + (kk & 3) * 32;
            mma_bf16_ss(tmem + ST_VN, make_sdesc_sw128(a, 16, 1024),
                        make_sdesc_sw128(slot + SL_W + kk * 2048, 8192, 1024), id_vn, kk > 0);
          }
          mma_commit(&bars[SB_VNFULL]);
          // O1^T = H^T Q^T into buffer ob (free once the epilogue read chunk c-2)
          if (c >= 2 && !mbar_wait(&bars[SB_OFREE + ob], ((c >> 1) & 1) ^ 1, abort_flag, err, 2u))
            break;
          tc_fence_after();
          for (int kk = 0; kk < ksteps_d; ++kk) {
            const uint32_t a = sbase + S_HT + (kk >> 2) * 16384 + (kk & 3) * 32;
            const uint32_t b = kq + (kk >> 2) * 16384 + 8192 + (kk & 3) * 32;
            mma_bf16_ss(tmem + ST_O1 + 64u * ob, make_sdesc_sw128(a, 16, 1024),
                        make_sdesc_sw128(b, 16, 1024), id_o1, kk > 0);
          }
          // H^T += Vns^T K ; O2^T = Vn^T Aqk^T
          if (!mbar_wait(&bars[SB_VNREADY], c & 1, abort_flag, err, 2u)) break;
          tc_fence_after();
          // H^T (already scaled by e^{G_C} in TMEM) += Vns^T K
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16_ss(tmem + ST_H, make_sdesc_sw128(sbase + S_VNS + kk * 32, 16, 1024),
                        make_sdesc_sw128(kq + kk * 2048, 16384, 1024), id_dh, 1);
          mma_commit(&bars[SB_DHFULL]);
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16_ss(tmem + ST_O2 + 64u * ob, make_sdesc_sw128(sbase + S_VN + kk * 32, 16, 1024),
                        make_sdesc_sw128(slot + SL_AQK + kk * 32, 16, 1024), id_o2, kk > 0);
          mma_commit(&bars[SB_OFULL + ob]);
          mma_commit(&bars[SB_KQE + st]);
          it_next(it, p, ustep);
        }
        mma_commit(&bars[SB_DRAIN]);
        mbar_wait(&bars[SB_DRAIN], 0, nullptr, err, 8u);
      }
      __syncwarp();
    } else if (warp < 4) {
      // ---------------- state warps: thread j owns row j of H^T, kept in TMEM
      // (f32, 128 columns at ST_H).  Per chunk: read H^T, write its bf16 copy
      // (the A operand of Vn and O1), write back e^{G_C} H^T so that the dH MMA
      // accumulates H_{c+1} = e^{G_C} H_c + dH in place.
      const int j = tid;
      const uint32_t lane_off = uint32_t(warp * 32) << 16;
      const uint32_t th = tmem + lane_off + ST_H;
      const bool jv = j < D;
      const int units = p.num_seqs * p.H_v;
      int c = 0;
      bool ok = true;
      for (int u = u0; u < units && ok; u += ustep) {
        const int n = u / p.H_v, h = u % p.H_v;
        int tb, te;
        seq_range(p, n, tb, te);
        const size_t state_off = (size_t(n) * p.H_v + h) * size_t(D) * D;
        const float* h0 = (p.h0 != nullptr && jv) ? p.h0 + state_off + j : nullptr;
        for (int t0 = tb; t0 < te && ok; t0 += C, ++c) {
          const int st = c & 1;
          const bool first = t0 == tb;
          if (!first) {  // H = e^{G_C} H_{c-1} + dH landed
            ok = mbar_wait(&bars[SB_DHFULL], (c - 1) & 1, abort_flag, err, 16u);
            if (!ok) break;
            tc_fence_after();
          }
          ok = mbar_wait_cluster(&bars[SB_SLOTF + st], (c >> 1) & 1, abort_flag, err, 16u);
          if (!ok) break;
          const float* sg = reinterpret_cast<const float*>(smem + S_SGATE) + st * SG_FLOATS;
          const float dec = sg[128];
#pragma unroll 1
          for (int q4 = 0; q4 < 4; ++q4) {
            float x[32];
            if (first) {
#pragma unroll
              for (int i = 0; i < 32; ++i)
                x[i] = (h0 != nullptr && 32 * q4 + i < D) ? h0[size_t(32 * q4 + i) * D] : 0.f;
            } else {
              tmem_ld32(th + 32u * q4, x);
              tmem_ld_wait();
            }
            const uint32_t ht = sbase + S_HT + (q4 >> 1) * 16384;
#pragma unroll
            for (int hc = 0; hc < 4; ++hc) {
              const int cc = 4 * (q4 & 1) + hc;
              st_shared_v4(ht + sw128_offset(j, cc * 16), pack_bf16x2(x[8 * hc], x[8 * hc + 1]),
                           pack_bf16x2(x[8 * hc + 2], x[8 * hc + 3]),
                           pack_bf16x2(x[8 * hc + 4], x[8 * hc + 5]),
                           pack_bf16x2(x[8 * hc + 6], x[8 * hc + 7]));
            }
#pragma unroll
            for (int i = 0; i < 32; ++i) x[i] *= dec;
            tmem_st32(th + 32u * q4, x);
          }
          tmem_st_wait();
          fence_proxy_async_smem();
          tc_fence_before();
          mbar_arrive(&bars[SB_HREADY]);
          // Vn = U - (H W)  ->  Vn^T and e^{G_C - G_r} Vn^T rows in bf16
          ok = mbar_wait(&bars[SB_VNFULL], c & 1, abort_flag, err, 16u);
          if (!ok) break;
          tc_fence_after();
          {
            const uint8_t* urow = smem + S_SLOT + st * SL_BYTES + SL_U;
#pragma unroll 1
            for (int q4 = 0; q4 < 4; ++q4) {  // 16 columns (two 16-byte chunks) at a time
              float vn[16];
              tmem_ld16(tmem + lane_off + ST_VN + 16u * q4, vn);
              tmem_ld_wait();
#pragma unroll
              for (int hc = 0; hc < 2; ++hc) {
                const int cc = 2 * q4 + hc;
                const uint4 uv = *reinterpret_cast<const uint4*>(urow + sw128_offset(j, cc * 16));
                const uint32_t uw[4] = {uv.x, uv.y, uv.z, uv.w};
                float x[8], y[8];
#pragma unroll
                for (int kq = 0; kq < 4; ++kq) {
                  x[2 * kq] = vn[8 * hc + 2 * kq] + __uint_as_float(uw[kq] << 16);
                  x[2 * kq + 1] = vn[8 * hc + 2 * kq + 1] + __uint_as_float(uw[kq] & 0xFFFF0000u);
                }
#pragma unroll
                for (int m = 0; m < 8; ++m) y[m] = x[m] * sg[64 + 8 * cc + m];
                st_shared_v4(sbase + S_VN + sw128_offset(j, cc * 16), pack_bf16x2(x[0], x[1]),
                             pack_bf16x2(x[2], x[3]), pack_bf16x2(x[4], x[5]),
                             pack_bf16x2(x[6], x[7]));
                st_shared_v4(sbase + S_VNS + sw128_offset(j, cc * 16), pack_bf16x2(y[0], y[1]),
                             pack_bf16x2(y[2], y[3]), pack_bf16x2(y[4], y[5]),
                             pack_bf16x2(y[6], y[7]));
              }
            }
          }
          fence_proxy_async_smem();
          tc_fence_before();
          mbar_arrive(&bars[SB_VNREADY]);
        }
        if (!ok) break;
        // final state: H after the last chunk's update (or h0 for an empty sequence)
        if (te > tb) {
          ok = mbar_wait(&bars[SB_DHFULL], (c - 1) & 1, abort_flag, err, 16u);
          if (!ok) break;
          tc_fence_after();
        }
        if (p.hT != nullptr && jv) {
          float* hT = p.hT + state_off + j;
#pragma unroll 1
          for (int q4 = 0; q4 < 4; ++q4) {
            float x[32];
            if (te > tb) {
              tmem_ld32(th + 32u * q4, x);
              tmem_ld_wait();
            } else {
#pragma unroll
              for (int i = 0; i < 32; ++i)
                x[i] = (h0 != nullptr && 32 * q4 + i < D) ? h0[size_t(32 * q4 + i) * D] : 0.f;
            }
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (32 * q4 + i < D) hT[size_t(32 * q4 + i) * D] = x[i];
          }
        }
        tc_fence_before();
      }
    } else {
      // ---------------- epilogue warps: o_r = e^{G_r} scale O1[r] + O2[r]
      const int e = tid - 128;
      const uint32_t lane_off = uint32_t((warp & 3) * 32) << 16;
      WgSync sync{&bars[SB_EPISYNC], 0};
      uint8_t* ost = smem + S_OST;
      const int row_bytes = D * 2;
      ChunkIter it;
      it_start(it, p, u0, ustep);
      while (it.ok) {
        const int c = it.c, ob = c & 1;
        const int L = min(C, it.te - it.t0);
        if (!mbar_wait(&bars[SB_OFULL + ob], (c >> 1) & 1, abort_flag, err, 128u)) break;
        tc_fence_after();
        if (!sync(abort_flag, err)) break;  // staging free (previous copy-out done)
        const float* sg = reinterpret_cast<const float*>(smem + S_SGATE) + ob * SG_FLOATS;
        const float sc = p.scale;
#pragma unroll 1
        for (int q4 = 0; q4 < 4; ++q4) {
          float o1[16], o2[16];
          tmem_ld16(tmem + lane_off + ST_O1 + 64u * ob + 16u * q4, o1);
          tmem_ld16(tmem + lane_off + ST_O2 + 64u * ob + 16u * q4, o2);
          tmem_ld_wait();
          if (e < D) {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const int r = 16 * q4 + i;
              const float val = fmaf(sg[r] * sc, o1[i], o2[i]);
              *reinterpret_cast<uint16_t*>(ost + r * row_bytes + 2 * e) =
                  __bfloat16_as_ushort(__float2bfloat16_rn(val));
            }
          }
        }
        tc_fence_before();
        mbar_arrive(&bars[SB_OFREE + ob]);
        // The slot of chunk c is no longer needed by anyone: hand it to the prep
        // group that fills it next.
        const int next_group = ((c >> 1) + 1) & 1;
        mbar_arrive_remote(
            mapa_shared(sbase + P_BARS + (PB_SLOTFREE + next_group) * 8, 1 + (c & 1)));
        if (!sync(abort_flag, err)) break;  // staging complete
        const int per_row = row_bytes / 16;
        for (int q = e; q < L * per_row; q += 128) {
          const int r = q / per_row, cc = q % per_row;
          const uint4 v = *reinterpret_cast<const uint4*>(ost + r * row_bytes + cc * 16);
          *reinterpret_cast<uint4*>(p.o + (size_t(it.t0 + r) * p.H_v + it.h) * D + cc * 8) = v;
        }
        it_next(it, p, ustep);
      }
    }
  } else {
    // =====================================================================
    // PREP (rank 1: even chunks, rank 2: odd chunks; group w takes every
    // other one of those)
    // =====================================================================
    const int par = int(rank) - 1;
    const uint32_t spine_slot = mapa_shared(sbase + S_SLOT + par * SL_BYTES, 0);
    const uint32_t spine_gate = mapa_shared(sbase + S_SGATE + par * SG_FLOATS * 4, 0);
    const uint32_t spine_slotf = mapa_shared(sbase + S_BARS + (SB_SLOTF + par) * 8, 0);
    if (warp == 8) {
      // ---------------- TMA: K, Q, V of each item into its group's buffers
      if (elect_one()) {
        ChunkIter it;
        it_start(it, p, u0, ustep);
        int last_k[2] = {-1, -1};
        while (it.ok) {
          const int c = it.c;
          if ((c & 1) == par) {
            const int w = (c >> 1) & 1, k = c >> 2;
            if (!mbar_wait(&bars[PB_KQVE + w], (k & 1) ^ 1, abort_flag, err, 1u)) break;
            uint64_t* fb = &bars[PB_KQVF + w];
            mbar_arrive_expect_tx(fb, uint32_t(nbox) * 3 * 8192);
            uint8_t* gsm = smem + w * P_WG;
            const int hk = it.h / (p.H_v / p.H_k);
            for (int b = 0; b < nbox; ++b) {
              tma_load_3d(gsm + P_KQ + b * 16384, &tm_k, fb, b * 64, hk, it.t0);
              tma_load_3d(gsm + P_KQ + b * 16384 + 8192, &tm_q, fb, b * 64, hk, it.t0);
              tma_load_3d(gsm + P_V + b * 8192, &tm_v, fb, b * 64, it.h, it.t0);
            }
            last_k[w] = k;
          }
          it_next(it, p, ustep);
        }
        for (int w = 0; w < 2; ++w)
          if (last_k[w] >= 0) mbar_wait(&bars[PB_KQVF + w], last_k[w] & 1, nullptr, err, 32u);
      }
      __syncwarp();
    } else if (warp == 9) {
      // ---------------- MMA issue for both groups, whichever is ready
      if (elect_one()) {
        const uint32_t id_p1 = make_idesc_bf16(128, 64, 0, 0);
        const uint32_t id_wu = make_idesc_bf16(128, 64, 1, 0);
        ChunkIter itp[2];
        int kp[2] = {0, 0}, kw[2] = {0, 0};
        for (int w = 0; w < 2; ++w) {
          it_start(itp[w], p, u0, ustep);
          it_align(itp[w], p, ustep, par + 2 * w);
        }
        long long last = clock64();
        while (true) {
          bool pending = false, prog = false;
          for (int w = 0; w < 2; ++w) {
            const uint32_t g = sbase + w * P_WG;
            const uint32_t tm = tmem + PT_WG * w;
            if (itp[w].ok) {
              pending = true;
              if (mbar_try_wait(&bars[PB_KQVF + w], kp[w] & 1) &&
                  (kp[w] == 0 || mbar_try_wait(&bars[PB_P1FREE + w], (kp[w] - 1) & 1))) {
                tc_fence_after();
                for (int kk = 0; kk < ksteps_d; ++kk) {
                  const uint32_t a = g + P_KQ + (kk >> 2) * 16384 + (kk & 3) * 32;
                  mma_bf16_ss(tm + PT_P1, make_sdesc_sw128(a, 16, 1024),
                              make_sdesc_sw128(a, 16, 1024), id_p1, kk > 0);
                }
                mma_commit(&bars[PB_P1F + w]);
                ++kp[w];
                it_next(itp[w], p, ustep);
                it_align(itp[w], p, ustep, par + 2 * w);
                prog = true;
              }
            }
            if (kw[w] < kp[w]) {
              pending = true;
              if (mbar_try_wait(&bars[PB_TREADY + w], kw[w] & 1)) {
                tc_fence_after();
                for (int kk = 0; kk < 4; ++kk)
                  mma_bf16_ss(tm + PT_W, make_sdesc_sw128(g + P_KQ + kk * 2048, 16384, 1024),
                              make_sdesc_sw128(g + P_T1B + kk * 32, 16, 1024), id_wu, kk > 0);
                for (int kk = 0; kk < 4; ++kk)
                  mma_bf16_ss(tm + PT_U, make_sdesc_sw128(g + P_V + kk * 2048, 8192, 1024),
                              make_sdesc_sw128(g + P_T2B + kk * 32, 16, 1024), id_wu, kk > 0);
                mma_commit(&bars[PB_KQVE + w]);
                mma_commit(&bars[PB_WUF + w]);
                ++kw[w];
                prog = true;
              }
            }
          }
          if (!pending || *abort_flag) break;
          if (prog) {
            last = clock64();
          } else if (clock64() - last > kSpinLimitCycles) {
            *abort_flag = 1;
            atomicOr(err, 2u);
            break;
          }
        }
        mma_commit(&bars[PB_DRAIN]);
        mbar_wait(&bars[PB_DRAIN], 0, nullptr, err, 8u);
      }
      __syncwarp();
    } else {
      // ---------------- prep groups: 128 threads each, one item at a time
      const int w = warp >> 2;
      const int pt = tid & 127;
      const uint32_t lane_off = uint32_t((warp & 3) * 32) << 16;
      uint8_t* gs = smem + w * P_WG;
      const uint32_t g = sbase + w * P_WG;
      float* Af = reinterpret_cast<float*>(gs + P_AF);
      float* Tf = reinterpret_cast<float*>(gs + P_TF);
      float* Xs = reinterpret_cast<float*>(gs + P_XS);
      float* gt = reinterpret_cast<float*>(gs + P_GATE);
      const uint32_t tm = tmem + PT_WG * w;
      WgSync sync{&bars[PB_SYNC + w], 0};
      ChunkIter it;
      it_start(it, p, u0, ustep);
      it_align(it, p, ustep, par + 2 * w);
      int k = 0;
      while (it.ok) {
        const int c = it.c;
        const int L = min(C, it.te - it.t0);
        const int h = it.h;
        // ---- gates of this chunk (padded rows: g = beta = 0)
        if (pt < 64) {
          const bool valid = pt < L;
          gt[PG_G + pt] = valid ? p.g[size_t(it.t0 + pt) * p.gb_stride + h] : 0.f;
          gt[PG_BET + pt] = valid ? p.beta[size_t(it.t0 + pt) * p.gb_stride + h] : 0.f;
        }
        if (!sync(abort_flag, err)) break;
        if (pt < 32) {  // inclusive scan of g over 64 rows (2 per lane)
          const float a0 = gt[PG_G + 2 * pt], a1 = gt[PG_G + 2 * pt + 1];
          float s = a0 + a1;
#pragma unroll
          for (int off = 1; off < 32; off <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, s, off);
            if (pt >= off) s += y;
          }
          const float excl = s - (a0 + a1);
          gt[PG_G + 2 * pt] = excl + a0;
          gt[PG_G + 2 * pt + 1] = excl + a0 + a1;
        }
        if (!sync(abort_flag, err)) break;
        {
          const float GC = gt[PG_G + 63];
          if (pt < 64) {
            const float Gr = gt[PG_G + pt];
            const float eg = __expf(Gr);
            gt[PG_EG + pt] = eg;
            gt[PG_ECG + pt] = __expf(GC - Gr);
            gt[PG_BEG + pt] = gt[PG_BET + pt] * eg;
            gt[PG_E1 + pt] = __expf(Gr - gt[PG_G + (pt & ~15)]);
          }
          for (int e = pt; e < 256; e += 128) {  // E2[b][s] = e^{G_{16b} - G_s}, s < 16b
            const int bb = e >> 6, s = e & 63;
            gt[PG_E2 + e] = (s < 16 * bb) ? __expf(gt[PG_G + 16 * bb] - gt[PG_G + s]) : 0.f;
          }
          if (pt == 0) gt[PG_DEC] = __expf(GC);
        }
        if (!sync(abort_flag, err)) break;
        // ---- P1 row pt: K K^T (pt < 64) or Q K^T (pt >= 64)
        if (!mbar_wait(&bars[PB_P1F + w], k & 1, abort_flag, err, 4u)) break;
        tc_fence_after();
        {
          float row[64];
          tmem_ld64(tm + lane_off + PT_P1, row);
          tc_fence_before();
          mbar_arrive(&bars[PB_P1FREE + w]);
          // row[s] *= e^{G_r - G_s} (s <= r): two factors <= 1 for the blocks of s
          // before r's 16-row block, a direct exponential inside it.
          const int r = pt & 63, rb = r >> 4;
          const float Gr = gt[PG_G + r];
          const float e1 = gt[PG_E1 + r];
          const float* e2 = gt + PG_E2 + 64 * rb;
#pragma unroll
          for (int sb = 0; sb < 4; ++sb) {
            if (sb < rb) {
#pragma unroll
              for (int jj = 0; jj < 16; ++jj) row[16 * sb + jj] *= e1 * e2[16 * sb + jj];
            } else if (sb == rb) {
#pragma unroll
              for (int jj = 0; jj < 16; ++jj) {
                const int s = 16 * sb + jj;
                row[s] = (s <= r) ? row[s] * __expf(Gr - gt[PG_G + s]) : 0.f;
              }
            } else {
#pragma unroll
              for (int jj = 0; jj < 16; ++jj) row[16 * sb + jj] = 0.f;
            }
          }
          if (pt < 64) {
            const float br = gt[PG_BET + r];
#pragma unroll
            for (int s = 0; s < 64; s += 4)
              *reinterpret_cast<float4*>(Af + r * kAS + s) =
                  make_float4(s + 0 < r ? br * row[s] : 0.f, s + 1 < r ? br * row[s + 1] : 0.f,
                              s + 2 < r ? br * row[s + 2] : 0.f, s + 3 < r ? br * row[s + 3] : 0.f);
          } else {
            const float sc = p.scale;
#pragma unroll
            for (int s = 0; s < 64; ++s) row[s] *= sc;
            uint32_t pk[32];
            pack_chunks<8>(row, pk);
            uint4* dst = reinterpret_cast<uint4*>(gs + P_AQK + r * 128);
#pragma unroll
            for (int cc = 0; cc < 8; ++cc)
              dst[cc] = make_uint4(pk[4 * cc], pk[4 * cc + 1], pk[4 * cc + 2], pk[4 * cc + 3]);
          }
        }
        if (!sync(abort_flag, err)) break;
        // ---- T = (I + A)^{-1}
        if (!invert_unit_lower64(Af, Tf, Xs, pt, sync, abort_flag, err)) break;
        // ---- T1 = T diag(beta e^G) (rows pt < 64), T2 = T diag(beta) (rows pt >= 64)
        {
          const int r = pt & 63;
          const float* scv = gt + (pt < 64 ? PG_BEG : PG_BET);
          float row[64];
#pragma unroll
          for (int s = 0; s < 64; s += 4) {
            const float4 t4 = *reinterpret_cast<const float4*>(Tf + r * kAS + s);
            const float4 s4 = *reinterpret_cast<const float4*>(scv + s);
            row[s] = s + 0 <= r ? t4.x * s4.x : 0.f;
            row[s + 1] = s + 1 <= r ? t4.y * s4.y : 0.f;
            row[s + 2] = s + 2 <= r ? t4.z * s4.z : 0.f;
            row[s + 3] = s + 3 <= r ? t4.w * s4.w : 0.f;
          }
          st_row64_bf16(g + (pt < 64 ? P_T1B : P_T2B), uint32_t(r), row);
        }
        fence_proxy_async_smem();
        mbar_arrive(&bars[PB_TREADY + w]);
        // ---- W^T, U^T, Aqk and the gate factors into the spine's slot
        // group 0 writes slot items 0, 2, 4 (the first needs no release), group 1
        // items 1, 3, 5 (each needs the release of the item before it)
        if (!mbar_wait_cluster(&bars[PB_SLOTFREE + w], (k + 1 + w) & 1, abort_flag, err, 4u))
          break;
        if (!mbar_wait(&bars[PB_WUF + w], k & 1, abort_flag, err, 4u)) break;
        tc_fence_after();
        {
          float row[64];
          uint32_t pk[32];
          tmem_ld64(tm + lane_off + PT_W, row);  // W^T row pt (d_k index)
          pack_chunks<8>(row, pk);
          st_row64_remote(spine_slot + SL_W, uint32_t(pt), pk);
          tmem_ld64(tm + lane_off + PT_U, row);  // U^T row pt (d_v index)
          pack_chunks<8>(row, pk);
          st_row64_remote(spine_slot + SL_U, uint32_t(pt), pk);
        }
        tc_fence_before();
        if (pt >= 64) {
          const uint4* src = reinterpret_cast<const uint4*>(gs + P_AQK + (pt - 64) * 128);
          uint32_t pk[32];
#pragma unroll
          for (int cc = 0; cc < 8; ++cc) {
            const uint4 v4 = src[cc];
            pk[4 * cc] = v4.x;
            pk[4 * cc + 1] = v4.y;
            pk[4 * cc + 2] = v4.z;
            pk[4 * cc + 3] = v4.w;
          }
          st_row64_remote(spine_slot + SL_AQK, uint32_t(pt - 64), pk);
        }
        if (pt < 33) {  // e^{G_r} [0, 64), e^{G_C - G_r} [64, 128), e^{G_C} at 128
          const float* src = gt + PG_EG + 4 * pt;  // PG_EG, PG_ECG, PG_DEC are contiguous
          st_cluster_v4(spine_gate + 16 * pt, __float_as_uint(src[0]), __float_as_uint(src[1]),
                        __float_as_uint(src[2]), __float_as_uint(src[3]));
        }
        fence_proxy_async_cluster();
        mbar_arrive_remote(spine_slotf);
        ++k;
        it_next(it, p, ustep);
        it_align(it, p, ustep, par + 2 * w);
      }
    }
  }

  // ---- teardown: wait for the whole cluster, then release TMEM
  tc_fence_before();
  __syncthreads();
  if (tid == 0) {
    const int exit_bar = spine ? SB_EXIT : PB_EXIT;
    mbar_arrive(&bars[exit_bar]);
    for (uint32_t r = 0; r < kCluster; ++r) {
      if (r == rank) continue;
      const uint32_t off = (r == 0 ? S_BARS + SB_EXIT * 8 : P_BARS + PB_EXIT * 8);
      mbar_arrive_remote(mapa_shared(sbase + off, r));
    }
    mbar_wait_cluster(&bars[exit_bar], 0, nullptr, err, 256u);
  }
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
  // As many clusters as can be resident at once (each cluster then walks its
  // share of the units), never more than there are units.
  static int max_clusters_cache[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  int max_clusters = (dev >= 0 && dev < 64) ? max_clusters_cache[dev] : 0;
  if (max_clusters <= 0) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(kCluster * (sm_count() / kCluster));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmemAlloc;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = kCluster;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    if (cudaOccupancyMaxActiveClusters(&max_clusters, prefill_kernel, &cfg) != cudaSuccess ||
        max_clusters <= 0) {
      cudaGetLastError();
      max_clusters = sm_count() / kCluster;
    }
    if (dev >= 0 && dev < 64) max_clusters_cache[dev] = max_clusters;
  }
  const int units = num_seqs * H_v;
  const int clusters = units < max_clusters ? units : max_clusters;
  prefill_kernel<<<clusters * kCluster, kThreads, kSmemAlloc, s>>>(tq, tk, tv, p);
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
