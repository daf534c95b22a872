// gdn_segmented.cu -- the segment-parallel (two-level) chunk scan.
//
// The chunk step of the state spine (page "ssm_gdn_tc_route.rs": the spine
// carries the f32 state across chunks) is affine in the state:
//     H  ->  (e^{G_C} I - K~^T W) H + K~^T U,
// so a run of chunks is one affine map  H -> M H + L  of its entry state.  A
// sequence cut into S segments of whole chunks can therefore be scanned in two
// levels instead of one chain of all its chunks:
//   A1  every segment but the last runs its chunks from a given entry: the
//       first from the caller's h0 (its outputs are final), the others from
//       zero, which leaves L_s (the state the segment adds) in its final state;
//   A2  every middle segment runs its chunks on v = 0 from H = I (the kernel's
//       identity-initial-state switch), which leaves M_s (the segment's
//       transition) in its final state;
//   C   entry(1) = L_0 (the first segment's true exit) and
//       entry(s + 1) = M_s entry(s) + L_s, a short sequential combine in f32;
//   B   every segment but the first runs again from its true entry state and
//       writes its outputs (and the last one the caller's hT).
// A1, A2 and B are launches of the ordinary chunk-parallel prefill kernel over
// segments (token ranges, per-segment state pointers, v read as zeros for
// A2).  Every chain is S times shorter, at the price of about three times the
// chunk work, which pays where the single-level scan leaves spines idle: few
// (sequence, head) units and long sequences, e.g. a tensor-parallel shard of
// a model holding a handful of heads per GPU.
//
// Segment s of a sequence with nc chunks covers chunks [s L, (s + 1) L),
// L = ceil(nc / S) (the last segments may be short or empty).
#include <cuda_runtime.h>

#include "gdn_internal.h"

namespace gdn {

namespace {

constexpr int kChunk = 64;

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

// Workspace layout of a segmented call (byte offsets, all 256-aligned).
struct SegLayout {
  size_t ring, segA1, segA2, segB, tabs, loc, trans, total;
};

SegLayout seg_layout(int num_seqs, int H_v, int D, int S) {
  SegLayout L;
  const size_t n1 = size_t(num_seqs) * (S - 1), n2 = size_t(num_seqs) * (S > 2 ? S - 2 : 1);
  const size_t state = size_t(H_v) * D * D * sizeof(float);
  size_t off = 0;
  L.ring = off;
  off += align256(prefill_ring_bytes(int(n1) * H_v));
  L.segA1 = off;
  off += align256(n1 * sizeof(int2));
  L.segA2 = off;
  off += align256(n2 * sizeof(int2));
  L.segB = off;
  off += align256(n1 * sizeof(int2));
  L.tabs = off;  // A1 h0, A1 hT, A2 h0, A2 hT, B h0, B hT: n1 pointers each
  off += align256(6 * n1 * sizeof(void*));
  L.loc = off;  // L_s of segments 0 .. S-2, overwritten in place by entry(s + 1)
  off += align256(n1 * state);
  L.trans = off;  // M_s of segments 1 .. S-2
  off += align256(n2 * state);
  L.total = off;
  return L;
}

// One CTA: the segment ranges and state-pointer tables of the three launches,
// from the device cu_seqlens.
__global__ void segment_plan_kernel(const int32_t* cu_seqlens, int num_seqs, int total_tokens,
                                    int S, int H_v, int D, const float* h0, float* hT,
                                    int2* segA1, int2* segA2, int2* segB, void** tabs,
                                    float* loc, float* trans) {
  const size_t state = size_t(H_v) * D * D;
  const size_t n1 = size_t(num_seqs) * (S - 1);
  // six tables of n1 state pointers (initial states are only read)
  float** a1_h0 = reinterpret_cast<float**>(tabs);
  float** a1_hT = reinterpret_cast<float**>(tabs + n1);
  float** a2_h0 = reinterpret_cast<float**>(tabs + 2 * n1);
  float** a2_hT = reinterpret_cast<float**>(tabs + 3 * n1);
  float** b_h0 = reinterpret_cast<float**>(tabs + 4 * n1);
  float** b_hT = reinterpret_cast<float**>(tabs + 5 * n1);
  for (int n = threadIdx.x; n < num_seqs; n += blockDim.x) {
    const int b = min(max(cu_seqlens[n], 0), total_tokens);
    const int e = min(max(cu_seqlens[n + 1], b), total_tokens);
    const int len = e - b;
    const int nc = (len + kChunk - 1) / kChunk;
    const int Lc = (nc + S - 1) / S;
    auto t = [&](int s) { return b + min(s * Lc * kChunk, len); };
    for (int s = 0; s < S - 1; ++s) {  // A1: segments 0 .. S-2
      const size_t i = size_t(n) * (S - 1) + s;
      segA1[i] = make_int2(t(s), t(s + 1));
      a1_h0[i] = (s == 0 && h0 != nullptr) ? const_cast<float*>(h0) + size_t(n) * state : nullptr;
      a1_hT[i] = loc + i * state;
    }
    for (int s = 1; s < S - 1; ++s) {  // A2: segments 1 .. S-2
      const size_t i = size_t(n) * (S - 2) + (s - 1);
      segA2[i] = make_int2(t(s), t(s + 1));
      a2_h0[i] = nullptr;  // the identity, by the launch's switch
      a2_hT[i] = trans + i * state;
    }
    for (int s = 1; s < S; ++s) {  // B: segments 1 .. S-1 from entry(s)
      const size_t i = size_t(n) * (S - 1) + (s - 1);
      segB[i] = make_int2(t(s), t(s + 1));
      b_h0[i] = loc + i * state;  // entry(s), left there by the combine
      b_hT[i] = (s == S - 1 && hT != nullptr) ? hT + size_t(n) * state : nullptr;
    }
  }
}

// entry(s + 1) = M_s entry(s) + L_s for s = 1 .. S-2, in place over L_s;
// entry(1) = L_0.  grid = (num_seqs * H_v, D / 16): CTA (unit, cb) owns
// columns 16 cb .. 16 cb + 15 of the unit's states (the columns of a state
// evolve independently), in f32.  Per step the CTA stages M_s in shared
// memory (rows padded by one float: conflict-free row-parallel reads) and
// thread t computes D / 16 consecutive columns of row t / (256 / D).
constexpr int kCombCols = 16;

template <int D>
__global__ void __launch_bounds__(256) segment_combine_kernel(int S, int H_v, float* loc,
                                                              const float* trans) {
  constexpr int CPT = D * kCombCols / 256;  // columns per thread: 8 (D = 128) or 4 (D = 64)
  extern __shared__ float cm[];             // Ms [D][D + 1], then E [D][kCombCols]
  float* Ms = cm;
  float* E = cm + D * (D + 1);
  const int unit = blockIdx.x, n = unit / H_v, h = unit % H_v, c0 = kCombCols * blockIdx.y;
  const size_t state = size_t(H_v) * D * D, head = size_t(h) * D * D;
  const int i = threadIdx.x / (kCombCols / CPT), cb = (threadIdx.x % (kCombCols / CPT)) * CPT;
  const float* L0 = loc + (size_t(n) * (S - 1)) * state + head;
  for (int idx = threadIdx.x; idx < D * kCombCols; idx += blockDim.x)
    E[idx] = L0[size_t(idx / kCombCols) * D + c0 + idx % kCombCols];
  for (int s = 1; s < S - 1; ++s) {
    const float* M = trans + (size_t(n) * (S - 2) + (s - 1)) * state + head;
    float* Ls = loc + (size_t(n) * (S - 1) + s) * state + head;
    for (int idx = threadIdx.x; idx < D * D / 4; idx += blockDim.x) {
      const float4 m = __ldg(reinterpret_cast<const float4*>(M) + idx);
      const int r = (4 * idx) / D, c = (4 * idx) % D;
      float* dst = Ms + r * (D + 1) + c;
      dst[0] = m.x;
      dst[1] = m.y;
      dst[2] = m.z;
      dst[3] = m.w;
    }
    __syncthreads();  // M staged; E holds entry(s)
    float acc[CPT];
#pragma unroll
    for (int j = 0; j < CPT; ++j) acc[j] = Ls[size_t(i) * D + c0 + cb + j];
#pragma unroll 4
    for (int k = 0; k < D; ++k) {
      const float m = Ms[i * (D + 1) + k];
      const float4* er = reinterpret_cast<const float4*>(E + k * kCombCols + cb);
#pragma unroll
      for (int j4 = 0; j4 < CPT / 4; ++j4) {
        const float4 e = er[j4];
        acc[4 * j4 + 0] = fmaf(m, e.x, acc[4 * j4 + 0]);
        acc[4 * j4 + 1] = fmaf(m, e.y, acc[4 * j4 + 1]);
        acc[4 * j4 + 2] = fmaf(m, e.z, acc[4 * j4 + 2]);
        acc[4 * j4 + 3] = fmaf(m, e.w, acc[4 * j4 + 3]);
      }
    }
    __syncthreads();  // every read of Ms and E for this step is done
#pragma unroll
    for (int j = 0; j < CPT; ++j) {
      E[i * kCombCols + cb + j] = acc[j];
      Ls[size_t(i) * D + c0 + cb + j] = acc[j];
    }
  }
}

}  // namespace

size_t prefill_segmented_workspace_bytes(int total_tokens, int num_seqs, int H_v, int D,
                                         int segments) {
  (void)total_tokens;
  if (segments < 2) return prefill_ring_bytes(num_seqs * H_v);
  return seg_layout(num_seqs, H_v, D, segments).total;
}

int prefill_auto_segments(int total_tokens, int num_seqs, int H_v) {
  // Two levels pay when the single-level launch leaves most spines idle and
  // the sequences are long: A1, A2 and B each run about nc / S chunk steps
  // per spine against nc for one level, but each launch also costs a fixed
  // start-up (the first ring entries, the last chunk's outputs) of some ten
  // chunk steps, and the combine S - 2 small products.  Measured on a B200
  // with 6 units: 4576 tokens (72 chunks) are faster in one level, so every
  // segment must span at least 24 chunks.
  const int units = num_seqs * H_v;
  const int budget = prefill_spine_budget();
  if (units <= 0 || units * 3 > budget) return 1;
  const int avg_chunks = (total_tokens / num_seqs + kChunk - 1) / kChunk;
  int S = budget / units + 1;  // units * (S - 1) <= budget
  if (S > 8) S = 8;
  if (S > avg_chunks / 24) S = avg_chunks / 24;
  return S >= 4 ? S : 1;
}

cudaError_t launch_prefill_segmented(const PrefillCall& c, int S, void* workspace,
                                     cudaStream_t s) {
  const SegLayout L = seg_layout(c.num_seqs, c.H_v, c.D, S);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int2* segA1 = reinterpret_cast<int2*>(ws + L.segA1);
  int2* segA2 = reinterpret_cast<int2*>(ws + L.segA2);
  int2* segB = reinterpret_cast<int2*>(ws + L.segB);
  void** tabs = reinterpret_cast<void**>(ws + L.tabs);
  float* loc = reinterpret_cast<float*>(ws + L.loc);
  float* trans = reinterpret_cast<float*>(ws + L.trans);
  const size_t n1 = size_t(c.num_seqs) * (S - 1);
  segment_plan_kernel<<<1, 256, 0, s>>>(c.cu_seqlens, c.num_seqs, c.total_tokens, S, c.H_v, c.D,
                                        c.h0, c.hT, segA1, segA2, segB, tabs, loc, trans);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;

  PrefillCall a1 = c;  // segments 0 .. S-2: L_s (and the first segment's outputs)
  a1.cu_seqlens = nullptr;
  a1.seg = segA1;
  a1.num_seqs = int(n1);
  a1.h0 = nullptr;
  a1.hT = nullptr;
  a1.h0_tab = reinterpret_cast<const float* const*>(tabs);
  a1.hT_tab = reinterpret_cast<float* const*>(tabs + n1);
  a1.workspace = ws + L.ring;
  if ((e = launch_prefill_call(a1, s)) != cudaSuccess) return e;

  if (S > 2) {
    PrefillCall a2 = a1;  // segments 1 .. S-2 on v = 0 from I: M_s
    a2.seg = segA2;
    a2.num_seqs = c.num_seqs * (S - 2);
    a2.h0_tab = reinterpret_cast<const float* const*>(tabs + 2 * n1);
    a2.hT_tab = reinterpret_cast<float* const*>(tabs + 3 * n1);
    a2.o = nullptr;
    a2.v_zero = 1;
    a2.h0_identity = 1;
    if ((e = launch_prefill_call(a2, s)) != cudaSuccess) return e;
    const int smem = int((c.D * (c.D + 1) + c.D * kCombCols) * sizeof(float));
    auto comb = c.D == 128 ? segment_combine_kernel<128> : segment_combine_kernel<64>;
    if ((e = cudaFuncSetAttribute(comb, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) !=
        cudaSuccess)
      return e;
    comb<<<dim3(c.num_seqs * c.H_v, c.D / kCombCols), 256, smem, s>>>(S, c.H_v, loc, trans);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }

  PrefillCall b = a1;  // segments 1 .. S-1 from their true entry states
  b.seg = segB;
  b.h0_tab = reinterpret_cast<const float* const*>(tabs + 4 * n1);
  b.hT_tab = reinterpret_cast<float* const*>(tabs + 5 * n1);
  b.o = c.o;
  b.v_zero = 0;
  return launch_prefill_call(b, s);
}

}  // namespace gdn
