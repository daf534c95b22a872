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
// One cluster of KS CTAs per 128 tokens, each CTA over its own K / KS slice
// (split-K, so that the 4576 x 5120 activation streams through ~all SMs).
// TMA streams 128x64 X tiles and Nx64 W tiles (128-byte swizzle) through a
// STAGES-deep mbarrier ring; one thread issues tcgen05.mma (M=128, N=N_pad,
// K=16 steps) into a TMEM accumulator.  Each CTA then stages its f32 partial
// in its own (now idle) pipeline shared memory; after a cluster barrier, rank
// r reduces rows r*128/KS .. of all KS partials in rank order (distributed
// shared memory reads, deterministic) and applies the gate epilogue in f32:
//   beta = sigmoid(ba),  gate = -exp(A_log) * softplus(ba + dt_bias).
// A second cluster barrier keeps every partial alive until it has been read.
// Every activation byte is read from HBM once; W (N*K*2 bytes) stays in L2.
// No multicast: each CTA loads its own tiles.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "gdn_device.cuh"
#include "gdn_internal.h"

namespace gdn {

__device__ uint32_t g_err_ba_gates;

constexpr int kBaBM = 128;       // tokens per CTA (MMA M)
constexpr int kBaBK = 64;        // K per TMA box (one 128-byte swizzle row)
constexpr int kBaNB = 2;         // boxes per pipeline stage: 2 x 128 contiguous bytes per row
constexpr int kBaMaxKS = 2;      // largest K split (CTAs per cluster): measured best
constexpr int kBaThreads = 128;  // 4 warps: TMA (warp 0), MMA (warp 1), all: epilogue

struct BaParams {
  const float* a_log;
  const float* dt_bias;
  float* out;
  int gate_stride, M, N, K, nv, vpg;
  int n_pad, stages, tmem_cols;
  int ks;  // CTAs per cluster (K split)
};

__device__ __forceinline__ float4 ld_cluster_f4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}

// Hardware cluster barrier; every thread of every CTA of the cluster reaches
// each call exactly once (no early exits in this kernel).
__device__ __forceinline__ void cluster_barrier() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}

__global__ void __launch_bounds__(kBaThreads, 1)
    ba_gates_kernel(const __grid_constant__ CUtensorMap tmap_x,
                    const __grid_constant__ CUtensorMap tmap_w, const BaParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const int stages = p.stages;
  const uint32_t a_box = kBaBM * 128, b_box = uint32_t(p.n_pad) * 128;
  const uint32_t a_bytes = kBaNB * a_box;
  const uint32_t b_bytes = kBaNB * b_box;
  uint8_t* a_s = smem;
  uint8_t* b_s = a_s + stages * a_bytes;
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(b_s + stages * b_bytes);
  uint64_t* empty_bar = full_bar + stages;
  uint64_t* done_bar = empty_bar + stages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const uint32_t warp = warp_id_sync();
  const uint32_t lane = threadIdx.x & 31;
  const int rank = int(cluster_ctarank());
  const int m0 = int(cluster_id_x()) * kBaBM;
  // K is split into boxes of kBaBK; this CTA owns boxes [kb_begin, kb_end),
  // consumed kBaNB boxes per pipeline stage (the last stage may be partial).
  const int kb_all = (p.K + kBaBK - 1) / kBaBK;
  const int kb_begin = kb_all * rank / p.ks, kb_end = kb_all * (rank + 1) / p.ks;
  const int nbox = kb_end - kb_begin;
  const int num_kb = (nbox + kBaNB - 1) / kBaNB;  // pipeline stages

  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    mbar_init(done_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmap_x);
    tma_prefetch_desc(&tmap_w);
  }
  if (warp == 0) tmem_alloc(tmem_slot, p.tmem_cols);
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (elect_one()) {  // TMA producer
      for (int kb = 0; kb < num_kb; ++kb) {
        const int s = kb % stages;
        const uint32_t ph = (kb / stages) & 1;
        if (!mbar_wait(&empty_bar[s], ph ^ 1, abort_flag, &g_err_ba_gates, 1u)) break;
        const int nb = min(kBaNB, nbox - kb * kBaNB);
        mbar_arrive_expect_tx(&full_bar[s], uint32_t(nb) * (a_box + b_box));
        for (int x = 0; x < nb; ++x) {
          const int kx = (kb_begin + kb * kBaNB + x) * kBaBK;
          tma_load_2d(a_s + s * a_bytes + x * a_box, &tmap_x, &full_bar[s], kx, m0);
          tma_load_2d(b_s + s * b_bytes + x * b_box, &tmap_w, &full_bar[s], kx, 0);
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (elect_one()) {  // MMA issuer
      const uint32_t idesc = make_idesc_bf16(kBaBM, p.n_pad, 0, 0);
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

  // Partial sums: warp w owns TMEM lanes 32w..32w+31 (tokens m0+32w+lane);
  // each row goes to the partial buffer P[128][n_pad + 4] f32 that reuses the
  // pipeline's shared memory (every MMA has completed once done_bar fired).
  const bool ok = num_kb == 0 || mbar_wait(done_bar, 0, abort_flag, &g_err_ba_gates, 4u);
  tc_fence_after();
  const int pstride = p.n_pad + 4;
  float* part = reinterpret_cast<float*>(smem);
  {
    float* prow = part + size_t(warp * 32 + lane) * pstride;
    for (int c = 0; c < p.n_pad; c += 16) {
      float acc[16];
      tmem_ld16(tmem + ((warp * 32u) << 16) + uint32_t(c), acc);
      tmem_ld_wait();
#pragma unroll
      for (int j = 0; j < 16; j += 4)
        *reinterpret_cast<float4*>(prow + c + j) =
            (ok && num_kb > 0) ? make_float4(acc[j], acc[j + 1], acc[j + 2], acc[j + 3])
                               : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
  tc_fence_before();
  cluster_barrier();  // every partial of the cluster is written
  // Reduction + epilogue: this CTA's rows r0 .. r0 + rows - 1; thread t takes
  // row r0 + t / tpr and a run of 4-column groups.
  {
    const int rows = kBaBM / p.ks;
    const int tpr = kBaThreads / rows;  // threads per row
    const int r = rank * rows + int(threadIdx.x) / tpr;
    const int m = m0 + r;
    const int group_dim = 2 * p.vpg;
    const uint32_t prow = smem_u32(part + size_t(r) * pstride);
    float* row = p.out + size_t(m) * p.gate_stride;
    for (int c = 4 * (int(threadIdx.x) % tpr); c < p.n_pad; c += 4 * tpr) {
      float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int q = 0; q < p.ks; ++q) {  // fixed order: deterministic
        const float4 v = ld_cluster_f4(mapa_shared(prow + uint32_t(c) * 4, uint32_t(q)));
        sum.x += v.x;
        sum.y += v.y;
        sum.z += v.z;
        sum.w += v.w;
      }
      const float acc[4] = {sum.x, sum.y, sum.z, sum.w};
      if (m < p.M && ok && !*abort_flag) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int n = c + j;
          if (n < p.N) {
            const int within = n % group_dim, grp = n / group_dim;
            const float ba = acc[j];
            if (within < p.vpg) {
              const int vh = grp * p.vpg + within;
              row[p.nv + vh] = 1.0f / (1.0f + __expf(-ba));
            } else {
              const int vh = grp * p.vpg + (within - p.vpg);
              const float z = ba + __ldg(&p.dt_bias[vh]);
              const float sp = fmaxf(z, 0.0f) + log1pf(__expf(-fabsf(z)));
              row[vh] = -__expf(__ldg(&p.a_log[vh])) * sp;
            }
          }
        }
      }
    }
  }
  cluster_barrier();  // no CTA leaves while its partial may still be read
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, p.tmem_cols);
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
  const int stage_bytes = kBaNB * (kBaBM * 128 + p.n_pad * 128);
  p.stages = (200 * 1024) / stage_bytes;
  if (p.stages > 6) p.stages = 6;
  if (p.stages < 2) p.stages = 2;
  // The pipeline buffers double as the f32 partial [128][n_pad + 4] afterwards.
  const size_t part_bytes = size_t(kBaBM) * (p.n_pad + 4) * 4;
  if (size_t(p.stages) * stage_bytes < part_bytes) return cudaErrorInvalidValue;
  const size_t smem = 1024 + size_t(p.stages) * stage_bytes + (2 * p.stages + 1) * 8 + 16;

  CUtensorMap tx, tw;
  {
    uint64_t dims[2] = {uint64_t(K), uint64_t(M)};
    uint64_t strides[1] = {uint64_t(k_stride) * 2};
    uint32_t box[2] = {uint32_t(kBaBK), uint32_t(kBaBM)};
    if (!encode_tmap_bf16(&tx, x, 2, dims, strides, box, true)) return cudaErrorInvalidValue;
  }
  {
    uint64_t dims[2] = {uint64_t(K), uint64_t(N)};
    uint64_t strides[1] = {uint64_t(K) * 2};
    uint32_t box[2] = {uint32_t(kBaBK), uint32_t(p.n_pad)};
    if (!encode_tmap_bf16(&tw, w, 2, dims, strides, box, true)) return cudaErrorInvalidValue;
  }
  cudaError_t e =
      cudaFuncSetAttribute(ba_gates_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  // K split: the largest power of two <= kBaMaxKS that keeps the grid within
  // the SMs and leaves every CTA at least one K box (KS = 2 for 4576 tokens).
  const int mtiles = (M + kBaBM - 1) / kBaBM;
  const int kb_all = (K + kBaBK - 1) / kBaBK;
  int ks = 1;
  while (ks < kBaMaxKS && mtiles * ks * 2 <= sm_count() && ks * 2 <= kb_all) ks *= 2;
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
  e = cudaLaunchKernelEx(&cfg, ba_gates_kernel, tx, tw, p);
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
