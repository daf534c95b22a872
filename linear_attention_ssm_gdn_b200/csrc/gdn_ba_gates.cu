// gdn_ba_gates.cu -- BA projection + gate epilogue on the tcgen05 tensor cores.
//
// Page "ssm_ba_gates_hopper.rs" (spark_model/layers/ops): every token's
// K-wide activation row is reduced against N = 2*nv rows of the BA weight;
// output n goes to the [gate(nv) | beta(nv)] row by ba_gates_slot.  The pages'
// kernels (the gb10 parent and the Hopper twin) do this on CUDA cores and read
// the row 96x resp. 12x; here it is a bf16 GEMM with f32 accumulation:
//
//   D[128 tokens x N] = X[128 x K] * W[N x K]^T
//
// One cluster of KS CTAs per BM tokens, each CTA over its own K / KS slice
// (split-K, so that the activation streams through ~all SMs): BM = 64 while
// the 64-row tiles in pairs fit the SMs in one wave (4576 tokens: 72 tiles x
// KS 2 = 144 CTAs), else 128; few tiles split K up to 8 ways.
// TMA streams BMx64 X tiles and Nx64 W tiles (128-byte swizzle) through a
// STAGES-deep mbarrier ring; one thread issues tcgen05.mma (M=BM, N=N_pad,
// K=16 steps) into a TMEM accumulator.  Rank r owns rows r*BM/KS .. of the
// tile: every CTA pushes each of its partial rows into the owner's receive
// buffer with distributed-shared-memory stores (no dependent remote loads),
// one cluster barrier publishes them, and the owner sums the KS partials of
// its rows in rank order (deterministic) from its own shared memory and
// applies the gate epilogue in f32, one output row at a time (coalesced):
//   beta = sigmoid(ba),  gate = -exp(A_log) * softplus(ba + dt_bias).
// Every activation byte is read from HBM once; W (N*K*2 bytes) stays in L2.
// No multicast: each CTA loads its own tiles.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "gdn_device.cuh"
#include "gdn_internal.h"

namespace gdn {

__device__ uint32_t g_err_ba_gates;

// tokens per CTA (MMA M): 64 while 64-row tiles in pairs fill the SMs, else 128
constexpr int kBaBK = 64;        // K per TMA box (one 128-byte swizzle row)
constexpr int kBaNB = 2;         // boxes per pipeline stage: 2 x 128 contiguous bytes per row
constexpr int kBaMaxKS = 8;      // largest K split (CTAs per cluster, the portable limit)
constexpr int kBaThreads = 512;  // TMA (warp 0), MMA (warp 1); all 16 warps: epilogue

struct BaParams {
  const float* a_log;
  const float* dt_bias;
  float* out;
  int gate_stride, M, N, K, nv, vpg;
  int n_pad, stages, tmem_cols;
  int ks;        // CTAs per cluster (K split)
  int overlay;   // 1: the receive buffer reuses the pipeline's shared memory
  uint32_t recv_off, const_off, bar_off;  // shared-memory layout (bytes)
};

constexpr uint32_t kBaMaxSmem = 232448;  // dynamic shared memory per CTA

__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_arrive_release() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait_acquire() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// log(1 + t) for t in [0, 1], relative error below 1e-5: the Taylor series
// t - t^2/2 + t^3/3 - ... through t^6 below t = 1/16 (truncation < t^6 / 7),
// and the fast logarithm of 1 + t above it (its absolute error over a result
// of at least log(17/16) = 0.06).
__device__ __forceinline__ float log1p_unit(float t) {
  if (t < 0.0625f)
    return t * (1.0f - t * (0.5f - t * (1.0f / 3.0f - t * (0.25f - t * (0.2f - t * (1.0f / 6.0f))))));
  return __logf(1.0f + t);
}

template <int BM>
__global__ void __launch_bounds__(kBaThreads, 1)
    ba_gates_kernel(const __grid_constant__ CUtensorMap tmap_x,
                    const __grid_constant__ CUtensorMap tmap_w, const BaParams p) {
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned start, kept as an offset from the __shared__ array so
  // that accesses through it stay shared-space (not generic) loads and stores
  uint8_t* smem = smem_raw + ((uint32_t(1024) - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const int stages = p.stages;
  const uint32_t a_box = BM * 128, b_box = uint32_t(p.n_pad) * 128;
  const uint32_t a_bytes = kBaNB * a_box;
  const uint32_t b_bytes = kBaNB * b_box;
  uint8_t* a_s = smem;
  uint8_t* b_s = a_s + stages * a_bytes;
  float* recv = reinterpret_cast<float*>(smem + p.recv_off);     // [KS][128 / KS][n_pad + 4]
  float* coef = reinterpret_cast<float*>(smem + p.const_off);    // -exp(A_log) [nv]
  float* dtb = coef + p.nv;                                       // dt_bias [nv]
  // output column j -> projection column n (bits 0-15) | v-head (16-30) | gate (31)
  uint32_t* colmap = reinterpret_cast<uint32_t*>(dtb + p.nv);
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + p.bar_off);
  uint64_t* empty_bar = full_bar + stages;
  uint64_t* done_bar = empty_bar + stages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const uint32_t warp = warp_id_sync();
  const uint32_t lane = threadIdx.x & 31;
  const int rank = int(cluster_ctarank());
  const int m0 = int(cluster_id_x()) * BM;
  // K is split into boxes of kBaBK; this CTA owns boxes [kb_begin, kb_end),
  // consumed kBaNB boxes per pipeline stage (the last stage may be partial).
  const int kb_all = (p.K + kBaBK - 1) / kBaBK;
  const int kb_begin = kb_all * rank / p.ks, kb_end = kb_all * (rank + 1) / p.ks;
  const int nbox = kb_end - kb_begin;
  const int num_kb = (nbox + kBaNB - 1) / kBaNB;  // pipeline stages
  // the first `stages` stages find their buffers free: issued during setup
  const int prologue = min(stages, num_kb);
  auto issue_stage = [&](int kb) {
    const int s = kb % stages;
    const int nb = min(kBaNB, nbox - kb * kBaNB);
    mbar_arrive_expect_tx(&full_bar[s], uint32_t(nb) * (a_box + b_box));
    for (int x = 0; x < nb; ++x) {
      const int kx = (kb_begin + kb * kBaNB + x) * kBaBK;
      tma_load_2d(a_s + s * a_bytes + x * a_box, &tmap_x, &full_bar[s], kx, m0);
      tma_load_2d(b_s + s * b_bytes + x * b_box, &tmap_w, &full_bar[s], kx, 0);
    }
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    mbar_init(done_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
    for (int kb = 0; kb < prologue; ++kb) issue_stage(kb);
  }
  if (warp == 0) tmem_alloc(tmem_slot, p.tmem_cols);
  for (int i = int(threadIdx.x); i < p.nv; i += kBaThreads) {
    coef[i] = -__expf(__ldg(&p.a_log[i]));
    dtb[i] = __ldg(&p.dt_bias[i]);
  }
  // Column j < nv is the gate of v-head j, column nv + h the beta of v-head h;
  // their projection outputs sit at n = (h / vpg) * 2 vpg + (vpg for the gate) + h % vpg.
  for (int j = int(threadIdx.x); j < 2 * p.nv; j += kBaThreads) {
    const bool is_gate = j < p.nv;
    const int vh = is_gate ? j : j - p.nv;
    const int n = (vh / p.vpg) * 2 * p.vpg + (is_gate ? p.vpg : 0) + vh % p.vpg;
    colmap[j] = uint32_t(n) | (uint32_t(vh) << 16) | (is_gate ? 0x80000000u : 0u);
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // With a separate receive buffer, the cluster barrier that publishes the
  // partials only needs every CTA of the cluster to have started: arrive now.
  if (!p.overlay) cluster_arrive_relaxed();

  if (warp == 0) {
    if (elect_one()) {  // TMA producer (the stages after the prologue)
      for (int kb = prologue; kb < num_kb; ++kb) {
        const int s = kb % stages;
        const uint32_t ph = (kb / stages) & 1;
        if (!mbar_wait(&empty_bar[s], ph ^ 1, abort_flag, &g_err_ba_gates, 1u)) break;
        issue_stage(kb);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (elect_one()) {  // MMA issuer
      const uint32_t idesc = make_idesc_bf16(BM, p.n_pad, 0, 0);
      bool ok = true;
      for (int kb = 0; kb < num_kb && ok; ++kb) {
        const int s = kb % stages;
        const uint32_t ph = (kb / stages) & 1;
        ok = mbar_wait(&full_bar[s], ph, abort_flag, &g_err_ba_gates, 2u);
        if (!ok) break;
        tc_fence_after();
        const int nb = min(kBaNB, nbox - kb * kBaNB);
        for (int x = 0; x < nb; ++x) {
          const uint32_t a0 = smem_u32(a_s + s * a_bytes + x * a_box);
          const uint32_t b0 = smem_u32(b_s + s * b_bytes + x * b_box);
#pragma unroll
          for (int j = 0; j < kBaBK / 16; ++j) {
            mma_bf16_ss(tmem, make_sdesc_sw128(a0 + j * 32, 16, 1024),
                        make_sdesc_sw128(b0 + j * 32, 16, 1024), idesc, (kb | x | j) != 0);
          }
        }
        mma_commit(&empty_bar[s]);
      }
      mma_commit(done_bar);  // fires once every issued MMA has completed
    }
    __syncwarp();
  }

  // Partial sums: warp w reads TMEM lane quadrant w % 4 (tile rows
  // BM/4 (w % 4) ..), column blocks of 16 from 16 (w / 4) in steps of 64.
  // Row r belongs to rank r / (BM / KS); this CTA's copy of it goes to slot
  // [my rank][r % (BM / KS)] of that rank's receive buffer.  When the buffer
  // reuses pipeline memory, every CTA of the cluster must be done with its
  // pipeline first (the barrier below is then a full one).
  const bool ok = num_kb == 0 || mbar_wait(done_bar, 0, abort_flag, &g_err_ba_gates, 4u);
  tc_fence_after();
  if (p.overlay) cluster_arrive_release();
  cluster_wait_acquire();  // every CTA of the cluster is running (and idle, overlaid)
  const int pstride = p.n_pad + 4;
  const int rows = BM / p.ks;
  // (M = 128: tile row r in TMEM lane r; M = 64: row r in lane r % 16 +
  // 32 (r / 16), so lanes 16..31 of each quadrant hold nothing: they take
  // part in the warp-wide TMEM loads and store nothing)
  {
    const uint32_t lq = warp & 3u;
    const bool holds = BM == 128 || lane < 16;
    const int r = int(lq) * (BM / 4) + (holds ? int(lane) : 0);
    const int owner = r / rows;
    const uint32_t dst = mapa_shared(
        smem_u32(recv + size_t(rank * rows + (r - owner * rows)) * pstride), uint32_t(owner));
    const bool live = ok && num_kb > 0;
    for (int c = 16 * int(warp >> 2); c < p.n_pad; c += 16 * (kBaThreads / 128)) {
      float acc[16];
      tmem_ld16(tmem + ((lq * 32u) << 16) + uint32_t(c), acc);
      tmem_ld_wait();
      if (holds) {
#pragma unroll
        for (int j = 0; j < 16; j += 4)
          st_cluster_v4(dst + uint32_t(c + j) * 4, live ? __float_as_uint(acc[j]) : 0u,
                        live ? __float_as_uint(acc[j + 1]) : 0u,
                        live ? __float_as_uint(acc[j + 2]) : 0u,
                        live ? __float_as_uint(acc[j + 3]) : 0u);
      }
    }
  }
  tc_fence_before();
  cluster_arrive_release();  // the pushes above, before the owners read them
  cluster_wait_acquire();
  // Reduction + epilogue over this rank's valid rows: a pass over the gate
  // columns (j < nv: the gate of v-head j) and one over the beta columns
  // (nv + j), each flat over (row lr, column j) so that consecutive threads
  // store consecutive columns of a row and no warp mixes the two paths;
  // (lr, j) advance by the fixed thread stride without divisions.
  if (ok && !*abort_flag) {
    const int nv = p.nv;
    const int row0 = m0 + rank * rows;
    const int total = max(0, min(rows, p.M - row0)) * nv;
    const int dl = kBaThreads / nv, dj = kBaThreads - dl * nv;
    const uint32_t qstride = uint32_t(rows * pstride);
#pragma unroll 1
    for (int pass = 0; pass < 2; ++pass) {
      int lr = int(threadIdx.x) / nv, j = int(threadIdx.x) - lr * nv;
      for (int i = int(threadIdx.x); i < total; i += kBaThreads) {
        const float* col = recv + uint32_t(lr * pstride) + (colmap[pass * nv + j] & 0xffffu);
        float sum = 0.0f;
        for (int q = 0; q < p.ks; ++q) sum += col[uint32_t(q) * qstride];  // rank order
        float val;
        if (pass == 0) {
          const float z = sum + dtb[j];
          val = coef[j] * (fmaxf(z, 0.0f) + log1p_unit(__expf(-fabsf(z))));
        } else {
          val = __frcp_rn(1.0f + __expf(-sum));
        }
        p.out[size_t(row0 + lr) * p.gate_stride + pass * nv + j] = val;
        lr += dl;
        j += dj;
        if (j >= nv) {
          j -= nv;
          ++lr;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, p.tmem_cols);
}

// ---------------------------------------------------------------------------
// Few tokens (the batched decode step: M = 1 .. kBaSmallM rows).
//
// Page "ssm_ba_gates_hopper.rs", module doc: one CTA per token starves the
// device when the step has few tokens (16 rows put 16 CTAs on the machine),
// hence its token-count guard.  Down to 9 tokens the tensor-core kernel above
// still fills enough SMs (one 64-row tile split 8 ways along K); at M <=
// kBaSmallM (measured: 8 tokens, 9 us, against 13 us there) these shapes
// split the OUTPUTS and the REDUCTION across CTAs instead of the tokens:
//   grid = NG output groups of kBaSmallNPB outputs x KS K slices, as clusters
//   of KS CTAs along K (one cluster per output group);
//   warp w of a CTA computes output n0 + w for every token of the chunk: each
//   lane holds 8 weights at a time and sweeps the token rows' matching 8
//   activations (16-byte loads; the activation slice is shared by the
//   group's 8 warps through L1), then a warp butterfly per token;
//   rank r of the cluster stores its [M_chunk x 8] partial sums into rank 0's
//   receive buffer (distributed shared memory), one cluster barrier publishes
//   them, and rank 0 adds the KS partials in rank order (deterministic) and
//   applies the gate epilogue of the large-M kernel.
// Tokens beyond kBaSmallMB per CTA go to further grid rows (blockIdx.y).  CUDA
// cores, f32 accumulation: at these sizes the weight read and the launch, not
// the arithmetic, set the time.
// ---------------------------------------------------------------------------
constexpr int kBaSmallM = 8;      // largest M sent to the few-token kernel (measured crossover)
constexpr int kBaSmallMB = 8;     // tokens per CTA row
constexpr int kBaSmallNPB = 8;    // outputs per CTA (one per warp)
constexpr int kBaSmallKS = 8;     // CTAs per cluster along K (portable cluster size)

struct BaSmallParams {
  const uint16_t* x;
  const uint16_t* w;
  const float* a_log;
  const float* dt_bias;
  float* out;
  int k_stride, gate_stride, M, N, K, nv, vpg, ks;
};

// MB: token rows per CTA (a power of two, the smallest >= M up to
// kBaSmallMB), so that no CTA carries predicated-off rows in its unrolled
// loops.
template <int MB>
__global__ void __launch_bounds__(32 * kBaSmallNPB, 1)
    ba_gates_small_kernel(const BaSmallParams p) {
  __shared__ float recv[kBaSmallKS][MB][kBaSmallNPB];
  const int rank = int(cluster_ctarank());
  const int grp = int(cluster_id_x());
  const int warp = int(threadIdx.x >> 5), lane = int(threadIdx.x & 31);
  const int m0 = int(blockIdx.y) * MB;
  const int mb = min(MB, p.M - m0);
  const int n = grp * kBaSmallNPB + warp;
  // K slice of this rank, in whole 8-column (16-byte) units
  const int units = p.K / 8;
  const int u0 = units * rank / p.ks, u1 = units * (rank + 1) / p.ks;
  // every CTA of the cluster is running before any remote store lands
  cluster_arrive_relaxed();
  cluster_wait_acquire();
  float acc[MB];
#pragma unroll
  for (int m = 0; m < MB; ++m) acc[m] = 0.0f;
  if (n < p.N) {
    const uint16_t* wrow = p.w + size_t(n) * p.K;
    constexpr int kUnrollU = MB >= 32 ? 1 : 2;  // two weight loads in flight, within registers
#pragma unroll kUnrollU
    for (int u = u0 + lane; u < u1; u += 32) {
      const uint4 wv = __ldg(reinterpret_cast<const uint4*>(wrow) + u);
      const uint32_t ww[4] = {wv.x, wv.y, wv.z, wv.w};
      float wf[8];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        wf[2 * e] = __uint_as_float(ww[e] << 16);
        wf[2 * e + 1] = __uint_as_float(ww[e] & 0xffff0000u);
      }
#pragma unroll
      for (int m = 0; m < MB; ++m) {
        if (m < mb) {
          const uint4 xv = __ldg(reinterpret_cast<const uint4*>(
                                     p.x + size_t(m0 + m) * p.k_stride) + u);
          const uint32_t xx[4] = {xv.x, xv.y, xv.z, xv.w};
          float a = acc[m];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            a = fmaf(wf[2 * e], __uint_as_float(xx[e] << 16), a);
            a = fmaf(wf[2 * e + 1], __uint_as_float(xx[e] & 0xffff0000u), a);
          }
          acc[m] = a;
        }
      }
    }
  }
  // per-token butterfly; lane 0 pushes the warp's column into rank 0
  const uint32_t base = mapa_shared(smem_u32(&recv[rank][0][warp]), 0u);
#pragma unroll
  for (int m = 0; m < MB; ++m) {
    if (m < mb) {
      float v = acc[m];
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
      if (lane == 0)
        asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(base + uint32_t(m * kBaSmallNPB) * 4),
                     "f"(v)
                     : "memory");
    }
  }
  cluster_arrive_release();
  cluster_wait_acquire();
  if (rank != 0) return;
  const int ng = min(kBaSmallNPB, p.N - grp * kBaSmallNPB);
  for (int i = int(threadIdx.x); i < mb * ng; i += 32 * kBaSmallNPB) {
    const int m = i / ng, j = i - m * ng;
    float sum = 0.0f;
    for (int q = 0; q < p.ks; ++q) sum += recv[q][m][j];  // rank order
    const int nn = grp * kBaSmallNPB + j;
    const int within = nn % (2 * p.vpg), g2 = nn / (2 * p.vpg);
    float val;
    int col;
    if (within < p.vpg) {  // beta of v-head g2 * vpg + within
      val = __frcp_rn(1.0f + __expf(-sum));
      col = p.nv + g2 * p.vpg + within;
    } else {               // gate of v-head g2 * vpg + within - vpg
      const int vh = g2 * p.vpg + within - p.vpg;
      const float z = sum + __ldg(&p.dt_bias[vh]);
      val = -__expf(__ldg(&p.a_log[vh])) * (fmaxf(z, 0.0f) + log1p_unit(__expf(-fabsf(z))));
      col = vh;
    }
    p.out[size_t(m0 + m) * p.gate_stride + col] = val;
  }
}

static cudaError_t launch_ba_gates_small(const uint16_t* x, int k_stride, const uint16_t* w,
                                         const float* a_log, const float* dt_bias, float* out,
                                         int gate_stride, int M, int N, int K, int nv, int vpg,
                                         cudaStream_t s) {
  BaSmallParams p;
  p.x = x;
  p.w = w;
  p.a_log = a_log;
  p.dt_bias = dt_bias;
  p.out = out;
  p.k_stride = k_stride;
  p.gate_stride = gate_stride;
  p.M = M;
  p.N = N;
  p.K = K;
  p.nv = nv;
  p.vpg = vpg;
  // K split: up to kBaSmallKS slices of at least 32 16-byte units each
  int ks = K / 8 / 32;
  ks = ks < 1 ? 1 : (ks > kBaSmallKS ? kBaSmallKS : ks);
  p.ks = ks;
  const int ngroups = (N + kBaSmallNPB - 1) / kBaSmallNPB;
  int mb = 1;
  while (mb < M && mb < kBaSmallMB) mb *= 2;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(ngroups * ks, (M + mb - 1) / mb);
  cfg.blockDim = dim3(32 * kBaSmallNPB);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeClusterDimension;
  attr.val.clusterDim.x = ks;
  attr.val.clusterDim.y = 1;
  attr.val.clusterDim.z = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  cudaError_t e;
  switch (mb) {
    case 1: e = cudaLaunchKernelEx(&cfg, ba_gates_small_kernel<1>, p); break;
    case 2: e = cudaLaunchKernelEx(&cfg, ba_gates_small_kernel<2>, p); break;
    case 4: e = cudaLaunchKernelEx(&cfg, ba_gates_small_kernel<4>, p); break;
    default: e = cudaLaunchKernelEx(&cfg, ba_gates_small_kernel<8>, p); break;
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

static int pow2_at_least(int x) {
  int c = 32;
  while (c < x) c <<= 1;
  return c;
}

cudaError_t launch_ba_gates(const uint16_t* x, int k_stride, const uint16_t* w,
                            const float* a_log, const float* dt_bias, float* out,
                            int gate_stride, int M, int N, int K, int nv, int vpg,
                            cudaStream_t s) {
  if (M == 0) return cudaSuccess;
  if (M <= kBaSmallM)
    return launch_ba_gates_small(x, k_stride, w, a_log, dt_bias, out, gate_stride, M, N, K, nv,
                                 vpg, s);
  BaParams p;
  p.a_log = a_log;
  p.dt_bias = dt_bias;
  p.out = out;
  p.gate_stride = gate_stride;
  p.M = M;
  p.N = N;
  p.K = K;
  p.nv = nv;
  p.vpg = vpg;
  p.n_pad = (N + 15) / 16 * 16;
  p.tmem_cols = pow2_at_least(p.n_pad);
  // Tile height: 64-row tiles in clusters of two while they fit the SMs in
  // one wave (4576 tokens: 72 tiles x 2 = 144 CTAs, each streaming 1/144 of
  // the activations), 128-row tiles beyond.
  const int kb_all = (K + kBaBK - 1) / kBaBK;
  const int BM = ((M + 63) / 64) * 2 <= sm_count() && kb_all >= 2 ? 64 : 128;
  // Layout: [stages][receive buffer, f32 [BM][n_pad + 4]][constants][barriers].
  // The receive buffer gets its own space when that still leaves two or more
  // stages, and otherwise reuses the (then idle) pipeline memory.
  const uint32_t stage_bytes = kBaNB * (uint32_t(BM) * 128 + uint32_t(p.n_pad) * 128);
  const uint32_t recv_bytes = uint32_t(BM) * (p.n_pad + 4) * 4;
  const uint32_t const_bytes = uint32_t(4 * nv) * 4;
  const uint32_t tail = const_bytes + 16 + (2 * 6 + 1) * 8 + 16;
  int stages = int((kBaMaxSmem - 1024 - recv_bytes - tail) / stage_bytes);
  p.overlay = stages < 2;
  if (p.overlay) stages = int((kBaMaxSmem - 1024 - tail) / stage_bytes);
  if (stages > 6) stages = 6;
  if (stages < 2) return cudaErrorInvalidValue;
  if (p.overlay && uint32_t(stages) * stage_bytes < recv_bytes) return cudaErrorInvalidValue;
  p.stages = stages;
  p.recv_off = p.overlay ? 0u : uint32_t(stages) * stage_bytes;
  p.const_off = (p.overlay ? uint32_t(stages) * stage_bytes : p.recv_off + recv_bytes);
  p.bar_off = (p.const_off + const_bytes + 15) / 16 * 16;
  const size_t smem = 1024 + p.bar_off + (2 * stages + 1) * 8 + 16;
  if (smem > kBaMaxSmem) return cudaErrorInvalidValue;

  CUtensorMap tx, tw;
  {
    uint64_t dims[2] = {uint64_t(K), uint64_t(M)};
    uint64_t strides[1] = {uint64_t(k_stride) * 2};
    uint32_t box[2] = {uint32_t(kBaBK), uint32_t(BM)};
    if (!encode_tmap_bf16(&tx, x, 2, dims, strides, box, true)) return cudaErrorInvalidValue;
  }
  {
    uint64_t dims[2] = {uint64_t(K), uint64_t(N)};
    uint64_t strides[1] = {uint64_t(K) * 2};
    uint32_t box[2] = {uint32_t(kBaBK), uint32_t(p.n_pad)};
    if (!encode_tmap_bf16(&tw, w, 2, dims, strides, box, true)) return cudaErrorInvalidValue;
  }
  auto kernel = BM == 64 ? ba_gates_kernel<64> : ba_gates_kernel<128>;
  cudaError_t e =
      cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  // K split: the largest power of two <= kBaMaxKS that keeps the grid within
  // the SMs and leaves every CTA at least one K box (KS = 2 for 4576 tokens).
  // Clusters of 4 and 8 only while few enough of them are placed at once
  // (at most ~33 clusters of 4 of these CTAs are resident together), so that
  // a few tiles still spread their K over many SMs.
  const int mtiles = (M + BM - 1) / BM;
  int ks = 1;
  while (ks < kBaMaxKS && mtiles * ks * 2 <= sm_count() && ks * 2 <= kb_all &&
         (ks < 2 || mtiles <= (ks == 2 ? 32 : 16)))
    ks *= 2;
  p.ks = ks;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(mtiles * ks);
  cfg.blockDim = dim3(kBaThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeClusterDimension;
  attr.val.clusterDim.x = ks;
  attr.val.clusterDim.y = 1;
  attr.val.clusterDim.z = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kernel, tx, tw, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// Read and clear this file's device error word (host; synchronous).
cudaError_t take_err_ba_gates(uint32_t* out) {
  uint32_t zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(out, g_err_ba_gates, sizeof(uint32_t));
  if (e != cudaSuccess) return e;
  return cudaMemcpyToSymbol(g_err_ba_gates, &zero, sizeof(uint32_t));
}

}  // namespace gdn
