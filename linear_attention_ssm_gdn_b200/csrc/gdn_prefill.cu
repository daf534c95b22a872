// gdn_prefill.cu -- chunk-parallel gated delta rule prefill on sm_100a.
//
// Page "ssm_gdn_tc_route.rs" names the piece this kernel replaces: the prefill
// "state spine" (chunk_delta_h) that carries the f32 recurrent state across
// chunks with bf16 tensor-core operands and an f32 accumulator.  Here the
// whole chunk step is one persistent kernel with one CTA per SM (a cooperative
// launch, so that every CTA is resident) in two roles:
//
//   SPINES (the first S CTAs) each own (sequence, v-head) units u = s, s+S, ...
//     and run their per-chunk critical chain on tcgen05 MMAs with TMEM
//     accumulators (M = d_v = 128 lanes), keeping H^T in registers (f32) and
//     its bf16 copy in TMEM as the A operand of the first MMA:
//       [Vn | -O1]^T = [U^T | 0] - H^T [W; Q]^T   (U^T preloaded by U^T I),
//       H^T <- e^{G_C} H^T + (e^{G_C - G_r} Vn)^T K   (Vn in bf16, from TMEM);
//     a separate output warpgroup forms  o_r = e^{G_r} scale O1_r + (Aqk Vn)_r
//     off that chain and stores it with TMA tensor stores;
//   PREPS (all other CTAs) compute everything that does not depend on H, for
//     chunk items of one spine each (prep p serves spine p % S and, with the
//     other preps of that spine, takes every n-th of its chunks), two items
//     at a time per CTA:
//       P1 = [K;Q] K^T                                 (MMA)
//       A[r][s]   = beta_r e^{G_r-G_s} k_r.k_s, s < r   (f32)
//       Aqk[r][s] = scale e^{G_r-G_s} q_r.k_s, s <= r
//       T = (I + A)^{-1}                   (blocked, f32; larger products TF32 MMA)
//       W^T = K^T (T diag(beta e^G))^T,  U^T = V^T (T diag(beta))^T   (MMAs)
//     and bulk-store W (row-major), U^T, Aqk (bf16) and the gate factors into the
//     owning spine's ring of kRing entries in the workspace (it stays in L2).
//   Hand-offs are release/acquire flags in the workspace: a prep publishes
//   entry j of spine s after its bulk store completed; the spine publishes that
//   it has copied the entry out, which frees it for item j + kRing.
//
// This is the WY/UT chunk form: within a chunk of rows r = 0..L-1 with
// G_r = g_0 + ... + g_r, (I + A) Vn = diag(beta) V - diag(beta e^G) K H, the
// outputs and the next state follow; the result equals the token recurrence up
// to rounding.  A chunk shorter than 64 rows gets g = beta = 0 in its padded
// rows, which then contribute nothing (exactly); padded rows are never stored.
// d_k = d_v = 64 runs the same code with the upper halves of every tile zero.
//
// No TMA multicast: every CTA loads its own K/Q/V tiles (L2 serves re-reads).
// Every wait is bounded (gdn_device.cuh): a timeout sets g_err_prefill and a
// grid-wide abort word, and every CTA then returns instead of waiting.  Named
// barriers are used only among threads that are all guaranteed to arrive.
//
// Progress: a spine consumes its chunks in order; each of its preps produces
// its share of them in order and only ever waits for that spine to free the
// ring entry of an older chunk, so the oldest unfinished chunk of every spine
// waits on nothing younger and the pipeline cannot deadlock while all CTAs
// are resident.
//
// Registers: 16 warps at 128 registers each; warps 0-7 (state warps, prep
// item groups) take 176 and warps 8-15 (single-thread roles, output warps)
// keep 80, each warpgroup changing its allocation at the top of its role.
#include <cuda.h>
#include <string.h>
#include <type_traits>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "gdn_device.cuh"
#include "gdn_internal.h"

namespace gdn {

__device__ uint32_t g_err_prefill;

namespace pf {

constexpr int C = 64;          // chunk rows
constexpr int kThreads = 512;  // 16 warps: 128 registers each at launch, re-allocated below
constexpr uint32_t kRegsWide = 176, kRegsNarrow = 80;  // warps 0-7 / warps 8-15
static_assert(2 * 128 * kRegsWide + 2 * 128 * kRegsNarrow == 128 * kThreads,
              "the re-allocated registers add up to the launch's allocation");
constexpr int kAS = 68;        // f32 row stride of the A / T scratch (16-byte rows)
constexpr int kRing = 8;       // ring entries per spine
constexpr int kMaxSpines = 256;
constexpr int kSpineSync = 288;  // the spine's per-chunk barriers: 8 state warps + the issuer warp
// Largest rise of the cumulative gate within a chunk (G_r - G_s, s <= r) that
// keeps every decay factor finite in f32 (e^88 overflows); a rise above it
// sets kErrGateRise in the prefill's device error word.
constexpr float kGateRise = 80.f;
constexpr uint32_t kErrGateRise = 64u;

// ---- ring entry (workspace): W (rows r, two 64-column d_k boxes) | U^T | Aqk | gate factors
constexpr uint32_t G_W = 0, G_U = 16384, G_AQK = 32768, G_GATE = 40960;
constexpr uint32_t G_GATE_BYTES = 528;  // e^{G_r} 64 | e^{G_C-G_r} 64 | e^{G_C} | pad
constexpr uint32_t SLOT_G = 41984;      // 41 KB, a multiple of 1024
// ---- flags (workspace head): one 64-byte line for the abort word, then one
// line per (spine, ring entry): ready count at +0, free count at +32 bytes.
constexpr uint32_t kFlagLine = 64;

// ---- spine shared memory (bytes from a 1024-aligned base): two chunk stages
// of STG_BYTES, each holding everything one chunk step reads, in two parts
// that are refilled independently:
//   part A: [box b: W rows 64x128B | Q rows 64x128B] x 2 (the N = 128 B
//           operand [W; Q]) and the gate factors -- read up to the [W; Q] MMA;
//   part B: K [box b: 64 x 128B] x 2, U^T [128 x 128B], Aqk [64 x 128B].
constexpr uint32_t STG_WQ = 0, STG_K = 32768, STG_U = 49152, STG_AQK = 65536, STG_GATE = 73728;
constexpr uint32_t STG_BYTES = 74752;  // 73 KB
constexpr uint32_t S_STG = 0;
constexpr uint32_t S_OT = S_STG + 2 * STG_BYTES;  // outputs, 2 chunks x 64 rows x d_v bf16
constexpr uint32_t S_VN = S_OT + 32768;           // two limbs: the low limb of H^T, bf16,
constexpr uint32_t S_VNS = S_VN + 16384;          //   [128 x 128B] per 64 d_k (S_VN, S_VNS)
constexpr uint32_t S_ID = S_VNS + 16384;          // the 64x64 identity, bf16 [64 x 128B]
constexpr uint32_t S_EG = S_ID + 8192;            // 4 x 64 f32: -scale e^{G_r} per chunk
constexpr uint32_t S_ECG = S_EG + 1024;           // 2 x 64 f32: e^{G_C - G_r} per chunk
constexpr uint32_t S_BARS = S_ECG + 512;
static_assert(S_OT % 1024 == 0 && STG_BYTES % 1024 == 0 && S_ID % 1024 == 0,
              "swizzled tiles are 1024-aligned");
static_assert(STG_GATE + G_GATE_BYTES <= STG_BYTES, "stage layout");
// ---- prep shared memory: two 128-thread item groups (item k: group k & 1)
// and three tile sets that rotate over the items (item k: set k % 3), so that
// one set is always being filled for the next item.  In a set, after P1 the Q
// boxes hold T diag(beta e^G) and T diag(beta) (bf16), and after the W/U MMAs
// [0, 32 KB) holds the item's W | U^T staging.
constexpr uint32_t P_SET = 49152;   // [box b: K 8K | Q 8K] x 2, V [box b: 8K] x 2
constexpr uint32_t P_KQ = 0, P_V = 32768;
constexpr uint32_t P_T1B = 8192, P_T2B = 24576;  // in the Q boxes, inside a set
constexpr uint32_t P_GRP = 3 * P_SET;            // the groups' own areas
constexpr uint32_t GA_AF = 0;                     // A, then T in place: f32 [64][kAS]
constexpr uint32_t GA_XS = GA_AF + 64 * kAS * 4;  // inverse scratch 32x32 f32
constexpr uint32_t GA_AQK = (GA_XS + 4096 + 1023) / 1024 * 1024;  // Aqk bf16 [64 x 128B]
constexpr uint32_t GA_GT = GA_AQK + 8192;         // 2 gate blocks
constexpr int PG_G = 0, PG_BET = 64, PG_E1 = 128, PG_E2 = 192, PG_BEG = 448, PG_EG = 512,
              PG_ECG = 576, PG_DEC = 640;  // floats; PG_EG..PG_DEC+3 is the published block
constexpr uint32_t PG_BYTES = 644 * 4;
constexpr uint32_t P_GS = (GA_GT + 2 * PG_BYTES + 1023) / 1024 * 1024;  // bytes per group
constexpr uint32_t P_BARS = P_GRP + 2 * P_GS;
constexpr uint32_t BAR_BYTES = 32 * 8;
constexpr uint32_t kMiscBytes = 16 + 4 * kMaxSpines;  // TMEM base, abort word, chunks per spine
constexpr uint32_t kSmemBytes =
    ((S_BARS > P_BARS ? S_BARS : P_BARS) + BAR_BYTES + kMiscBytes + 15) / 16 * 16;
constexpr uint32_t kSmemAlloc = kSmemBytes + 1024;
static_assert(kSmemAlloc <= 232448, "shared memory budget");
static_assert(S_BARS % 8 == 0 && P_BARS % 8 == 0, "barrier alignment");
static_assert(P_V == 32768 && G_U == 16384 && G_AQK == 32768 && P_SET >= P_V + 8192,
              "W | U^T | Aqk staging mirrors the ring entry");
static_assert((GA_GT + PG_EG * 4) % 16 == 0 && (GA_GT + PG_BYTES + PG_EG * 4) % 16 == 0 &&
                  P_GS % 16 == 0, "gate blocks are bulk-copy sources");
static_assert(P_SET % 1024 == 0 && P_GRP % 1024 == 0 && P_GS % 1024 == 0 && GA_AQK % 1024 == 0,
              "swizzled tiles");

// ---- barriers (spine)
enum {
  SB_AF = 0,       // +stage: part A landed: Q (TMA), W and the gate factors (bulk)
  SB_AE = 2,       // +stage: part A free: the [W; Q] MMA is done (commit)
  SB_BF = 4,       // +stage: part B landed: K (TMA), U^T and Aqk (bulk)
  SB_BE = 6,       // +stage: part B free: dH and O2 are done (commit)
  SB_VOFULL = 8,   // H^T [W; Q]^T done (commit)
  SB_DHFULL = 9,   // dH = Vns^T K done (commit)
  SB_OFULL = 10,   // +buf: O2 (and so O1) done (commit)
  SB_DRAIN = 12,
  SB_OEMPTY = 13,  // +buf: the output warps have read O1 / O2 of the chunk and zeroed
                   // the O1 half (1; once more at start-up)
  SB_COUNT = 15
};
// ---- barriers (prep).  Item k: group g = k & 1, kg = k >> 1 its index in
// the group, tile set k % 3, P1 buffer and gate block kg & 1 of group g.
enum {
  PB_KQVF = 0,     // +set: K, Q, V tiles landed (TMA)
  PB_STORED = 3,   // +set: the item's staging, Aqk and gates read by the bulk store (1)
  PB_P1F = 6,      // +2g+buf: P1 = [K;Q] K^T done (commit)
  PB_P1FREE = 10,  // +2g+buf: P1 read back (128)
  PB_TREADY = 14,  // +g: T1, T2 written (128)
  PB_WUF = 16,     // +g: W^T, U^T done (commit)
  PB_GATEF = 18,   // +2g+buf: gate block written (32, the loader warp)
  PB_STAGED = 22,  // +g: W | U^T staged (1)
  PB_DRAIN = 24,
  PB_GBFREE = 25,  // +2g+buf: gate block read by the bulk store (1, the store warp)
  PB_COUNT = 29
};
static_assert(int(PB_COUNT) <= 32 && int(SB_COUNT) <= 32, "barrier area");

// ---- TMEM columns
// spine: [Vn^T | -O1^T] x2 (128 columns each; the Vn half ends as bf16 Vn,
// Vns), O2^T (64), the bf16 copy of H^T (64), dH^T (lane j = d_v row j)
constexpr uint32_t ST_VO = 0, ST_O2 = 256, ST_HT = 320, ST_DH = 384;
constexpr uint32_t PT_W = 128, PT_U = 192, PT_WG = 256;  // prep, per group: P1 x2 at 0, 64

struct Params {
  const float* g;
  const float* beta;
  const int32_t* cu_seqlens;
  const float* h0;
  float* hT;
  uint16_t* o;  // NULL: outputs not stored
  // Optional per-sequence overrides (the segment-parallel scan runs the
  // kernel over segments of the caller's sequences): token ranges [x, y),
  // initial-state and final-state pointers ([H_v, D, D] each; NULL entry =
  // zeros / not stored), and v read as zeros.
  const int2* seg;
  const float* const* h0_tab;
  float* const* hT_tab;
  int v_zero;
  int h0_identity;  // 1: every initial state is the identity (needs d_k == d_v)
  uint32_t* flags;  // abort line + S * kRing flag lines
  uint8_t* ring;    // S * kRing entries of SLOT_G bytes
  int gb_stride, num_seqs, total_tokens, H_k, H_v, D;
  int S;  // spine CTAs: blockIdx.x < S; the others are preps
  float scale;
  // cycles a pipeline wait polls before it gives up (drains of in-flight
  // copies and MMAs before exit always use the full kSpinLimitCycles)
  long long spin_limit;
};

__device__ __forceinline__ uint32_t* ready_flag(const Params& p, int s, int e) {
  return p.flags + (1 + s * kRing + e) * (kFlagLine / 4);
}
__device__ __forceinline__ uint32_t* free_flag(const Params& p, int s, int e) {
  return ready_flag(p, s, e) + 8;
}
__device__ __forceinline__ uint8_t* ring_entry(const Params& p, int s, int e) {
  return p.ring + size_t(s * kRing + e) * SLOT_G;
}

template <bool kSeg>
__device__ __forceinline__ void seq_range(const Params& p, int n, int& b, int& e) {
  if (kSeg && p.seg != nullptr) {
    const int2 r = p.seg[n];
    b = min(max(r.x, 0), p.total_tokens);
    e = min(max(r.y, b), p.total_tokens);
    return;
  }
  b = min(max(p.cu_seqlens[n], 0), p.total_tokens);
  e = min(max(p.cu_seqlens[n + 1], b), p.total_tokens);
}

template <bool kSeg>
__device__ __forceinline__ int unit_chunks(const Params& p, int u) {
  int b, e;
  seq_range<kSeg>(p, u / p.H_v, b, e);
  return (e - b + C - 1) / C;
}

// Walks the chunks of the units a spine owns (u = s, s + S, ...); `c` counts
// chunks over all of them.
struct ChunkIter {
  int u, n, h, t0, tb, te, c;
  bool ok;
};

template <bool kSeg>
__device__ __forceinline__ void it_load_unit(ChunkIter& it, const Params& p) {
  it.n = it.u / p.H_v;
  it.h = it.u % p.H_v;
  seq_range<kSeg>(p, it.n, it.tb, it.te);
  it.t0 = it.tb;
}

template <bool kSeg>
__device__ __forceinline__ void it_skip_empty(ChunkIter& it, const Params& p) {
  const int units = p.num_seqs * p.H_v;
  while (it.ok && it.t0 >= it.te) {
    it.u += p.S;
    if (it.u >= units) {
      it.ok = false;
      break;
    }
    it_load_unit<kSeg>(it, p);
  }
}

template <bool kSeg>
__device__ __forceinline__ void it_start(ChunkIter& it, const Params& p, int s) {
  it.u = s;
  it.c = 0;
  it.ok = s < p.num_seqs * p.H_v;
  if (it.ok) it_load_unit<kSeg>(it, p);
  it_skip_empty<kSeg>(it, p);
}

template <bool kSeg>
__device__ __forceinline__ void it_next(ChunkIter& it, const Params& p) {
  it.t0 += C;
  ++it.c;
  it_skip_empty<kSeg>(it, p);
}

// The items of one prep CTA: global item i = j * S + s (chunk j of spine s),
// i = prank, prank + Pn, ...; k counts the valid ones (k & 1 picks the group).
struct PrepIter {
  int i, k, s, j, h, t0, L, stride;
  bool ok;
};

// Prep CTA prank serves one spine, s = prank % S, together with the other
// preps of the same residue: the n = ceil((Pn - s) / S) of them take its
// chunks j = prank / S, + n, + 2n, ...  A prep that waits for a free ring
// entry of its spine therefore never holds back another spine's items.
template <bool kSeg>
__device__ __forceinline__ bool pi_fill(PrepIter& it, const Params& p, const int* sJ, int iend) {
  (void)iend;
  const int s = it.s;
  if (it.i < sJ[s]) {
    const int units = p.num_seqs * p.H_v;
    int jj = it.i;
    for (int u = s; u < units; u += p.S) {
      const int nc = unit_chunks<kSeg>(p, u);
      if (jj < nc) {
        int tb, te;
        seq_range<kSeg>(p, u / p.H_v, tb, te);
        it.j = it.i;
        it.h = u % p.H_v;
        it.t0 = tb + jj * C;
        it.L = min(C, te - it.t0);
        return true;
      }
      jj -= nc;
    }
  }
  return false;
}

template <bool kSeg>
__device__ __forceinline__ void pi_start(PrepIter& it, const Params& p, const int* sJ, int iend,
                                         int prank) {
  const int pn = int(gridDim.x) - p.S;
  it.s = prank % p.S;
  it.i = prank / p.S;
  it.stride = (pn - it.s + p.S - 1) / p.S;
  it.k = 0;
  it.ok = pi_fill<kSeg>(it, p, sJ, iend);
}

template <bool kSeg>
__device__ __forceinline__ void pi_next(PrepIter& it, const Params& p, const int* sJ, int iend) {
  it.i += it.stride;
  ++it.k;
  it.ok = pi_fill<kSeg>(it, p, sJ, iend);
}

template <bool kSeg>
__device__ __forceinline__ void pi_align(PrepIter& it, const Params& p, const int* sJ, int iend,
                                         int w) {
  while (it.ok && (it.k & 1) != w) pi_next<kSeg>(it, p, sJ, iend);
}

// The low bf16 limb of 64 f32 values: x - bf16(x) (exact in f32), rounded to
// bf16, as one 128-byte row of a 128B-swizzled tile (the second limb of the
// state copy).
__device__ __forceinline__ void st_row64_bf16_lo(uint32_t tile, uint32_t row, const float* x) {
  float r[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) {
#pragma unroll
    for (int e = 0; e < 8; ++e)
      r[e] = x[8 * c + e] - __bfloat162float(__float2bfloat16_rn(x[8 * c + e]));
    st_shared_v4(tile + sw128_offset(row, c * 16), pack_bf16x2(r[0], r[1]), pack_bf16x2(r[2], r[3]),
                 pack_bf16x2(r[4], r[5]), pack_bf16x2(r[6], r[7]));
  }
}

// ---------------------------------------------------------------------------
// T = (I + A)^{-1} in place: on entry M holds the strictly lower triangular
// 64x64 A (f32, row stride kAS, zeros on and above the diagonal), on exit the
// unit lower triangular T.  128 threads (4 warps), 16x16 blocks
// D_i = (I + A_ii)^{-1}:
//   1. warp w: D_w by forward substitution (lane j < 16 owns column j and
//      pushes each new x_l into the running sums of the rows below it), then
//      written over A_ww;
//   2. warp pair p (blocks 2p, 2p+1): T_{2p+1,2p} = -D_{2p+1} A_{2p+1,2p} D_{2p},
//      written over A_{2p+1,2p} once the pair has read it;
//   3. X = A[32:64, 0:32] T[0:32, 0:32];
//   4. T[32:64, 0:32] = -T[32:64, 32:64] X, written over A[32:64, 0:32].
// Steps 2, 3 and 4 (most of the arithmetic) run on the tensor cores as
// warp-level m16n8k8 products with TF32 inputs and f32 accumulation (steps 3
// and 4: each warp a 16x16 output tile; step 2: each warp 16 rows x 8
// columns): they read a quarter of the shared memory that CUDA-core tiles
// would, and shared memory is what two item groups on one SM compete for (a
// probe: 5371 -> 3781 cycles per inverse with both groups busy, steps 3 and
// 4).  TF32 keeps 10 mantissa bits, and T is rounded to bf16 (8 bits) right
// after; on random inputs T differs from the f32 products by 7e-5 relative.  The upper blocks stay the zeros of A.  bar_base: named barrier
// ids bar_base (128 threads), bar_base+1+p (pairs).  X and the pair products
// use the 32x32 f32 scratch Xs.
// ---------------------------------------------------------------------------
// TF32 tensor-core products inside the blocked inverse: f32 -> tf32 (round
// to nearest) and one warp-level m16n8k8 MMA with f32 accumulation.  The
// fragments: A (16x8) a0 = (g, t), a1 = (g+8, t), a2 = (g, t+4), a3 = (g+8, t+4);
// B (8x8) b0 = (t, g), b1 = (t+4, g); D (16x8) d0/d1 = (g, 2t / 2t+1), d2/d3 =
// (g+8, 2t / 2t+1), with g = lane / 4 and t = lane % 4.
__device__ __forceinline__ uint32_t f2tf32(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return r;
}
__device__ __forceinline__ void mma_tf32_16x8x8(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                                uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void invert_unit_lower64(float* M, float* Xs, int p, int bar_base) {
  const int w = p >> 5, ln = p & 31;
  // 1. diagonal blocks
  {
    float x[16];
    const int j = ln;
    if (ln < 16) {
      const float* Ab = M + (16 * w) * kAS + 16 * w;
      float acc[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) acc[i] = 0.f;
#pragma unroll
      for (int l = 0; l < 16; ++l) {
        x[l] = (l < j) ? 0.f : ((l == j) ? 1.f : -acc[l]);
#pragma unroll
        for (int i = l + 1; i < 16; ++i) acc[i] = fmaf(Ab[i * kAS + l], x[l], acc[i]);
      }
    }
    __syncwarp();  // every lane has read A_ww
    if (ln < 16) {
      float* Tb = M + (16 * w) * kAS + 16 * w + j;
#pragma unroll
      for (int i = 0; i < 16; ++i) Tb[i * kAS] = x[i];
    }
  }
  // 2. first sub-diagonal blocks, one per warp pair (blocks 2p, 2p+1), on
  //    the tensor cores like steps 3 and 4: warp 2p + h computes columns
  //    8 h .. 8 h + 7 of Y = A_{2p+1,2p} D_{2p} (into the pair's scratch),
  //    then of -D_{2p+1} Y over A_{2p+1,2p} once the pair has read it
  {
    const int pr = w >> 1, h = w & 1;
    const int bi = 2 * pr + 1, bj = 2 * pr;
    const int gq = ln >> 2, tq = ln & 3;
    float* Y = Xs + pr * 256;  // 16 x 16, row stride 16
    named_sync(bar_base + 1 + pr, 64);
    float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int k0 = 0; k0 < 16; k0 += 8) {
      const float* ab = M + (16 * bi) * kAS + 16 * bj + k0;
      const float* bb = M + (16 * bj + k0) * kAS + 16 * bj + 8 * h;
      mma_tf32_16x8x8(d, f2tf32(ab[gq * kAS + tq]), f2tf32(ab[(gq + 8) * kAS + tq]),
                      f2tf32(ab[gq * kAS + tq + 4]), f2tf32(ab[(gq + 8) * kAS + tq + 4]),
                      f2tf32(bb[tq * kAS + gq]), f2tf32(bb[(tq + 4) * kAS + gq]));
    }
    *reinterpret_cast<float2*>(Y + gq * 16 + 8 * h + 2 * tq) = make_float2(d[0], d[1]);
    *reinterpret_cast<float2*>(Y + (gq + 8) * 16 + 8 * h + 2 * tq) = make_float2(d[2], d[3]);
    named_sync(bar_base + 1 + pr, 64);  // Y complete, A_{2p+1,2p} read by the pair
    float z[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int k0 = 0; k0 < 16; k0 += 8) {
      const float* ab = M + (16 * bi) * kAS + 16 * bi + k0;
      const float* yb = Y + k0 * 16 + 8 * h;
      mma_tf32_16x8x8(z, f2tf32(ab[gq * kAS + tq]), f2tf32(ab[(gq + 8) * kAS + tq]),
                      f2tf32(ab[gq * kAS + tq + 4]), f2tf32(ab[(gq + 8) * kAS + tq + 4]),
                      f2tf32(yb[tq * 16 + gq]), f2tf32(yb[(tq + 4) * 16 + gq]));
    }
    float* tb = M + (16 * bi) * kAS + 16 * bj + 8 * h + 2 * tq;
    *reinterpret_cast<float2*>(tb + gq * kAS) = make_float2(-z[0], -z[1]);
    *reinterpret_cast<float2*>(tb + (gq + 8) * kAS) = make_float2(-z[2], -z[3]);
  }
  named_sync(bar_base, 128);
  // 3. X = A[32:64, 0:32] T[0:32, 0:32] and 4. T[32:64, 0:32] = -T[32:64, 32:64] X
  //    on the tensor cores (m16n8k8, TF32 inputs, f32 accumulate): warp w
  //    computes rows 16 (w >> 1) .., columns 16 (w & 1) .. of each product
  const int wq = p >> 5, gq = (p & 31) >> 2, tq = p & 3;
  const int mr = 16 * (wq >> 1), ncol = 16 * (wq & 1);
  {
    float d[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
    for (int k0 = 0; k0 < 32; k0 += 8) {
      const float* ab = M + (32 + mr) * kAS + k0;
      const uint32_t a0 = f2tf32(ab[gq * kAS + tq]), a1 = f2tf32(ab[(gq + 8) * kAS + tq]);
      const uint32_t a2 = f2tf32(ab[gq * kAS + tq + 4]), a3 = f2tf32(ab[(gq + 8) * kAS + tq + 4]);
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        const float* bb = M + k0 * kAS + ncol + 8 * nt;
        mma_tf32_16x8x8(d[nt], a0, a1, a2, a3, f2tf32(bb[tq * kAS + gq]), f2tf32(bb[(tq + 4) * kAS + gq]));
      }
    }
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      const int cc = ncol + 8 * nt + 2 * tq;
      *reinterpret_cast<float2*>(Xs + (mr + gq) * 32 + cc) = make_float2(d[nt][0], d[nt][1]);
      *reinterpret_cast<float2*>(Xs + (mr + gq + 8) * 32 + cc) = make_float2(d[nt][2], d[nt][3]);
    }
  }
  named_sync(bar_base, 128);  // A[32:64, 0:32] read, X complete
  {
    float d[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
    for (int k0 = 0; k0 < 32; k0 += 8) {
      const float* ab = M + (32 + mr) * kAS + 32 + k0;
      const uint32_t a0 = f2tf32(ab[gq * kAS + tq]), a1 = f2tf32(ab[(gq + 8) * kAS + tq]);
      const uint32_t a2 = f2tf32(ab[gq * kAS + tq + 4]), a3 = f2tf32(ab[(gq + 8) * kAS + tq + 4]);
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        const float* bb = Xs + k0 * 32 + ncol + 8 * nt;
        mma_tf32_16x8x8(d[nt], a0, a1, a2, a3, f2tf32(bb[tq * 32 + gq]), f2tf32(bb[(tq + 4) * 32 + gq]));
      }
    }
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      const int cc = ncol + 8 * nt + 2 * tq;
      *reinterpret_cast<float2*>(M + (32 + mr + gq) * kAS + cc) = make_float2(-d[nt][0], -d[nt][1]);
      *reinterpret_cast<float2*>(M + (32 + mr + gq + 8) * kAS + cc) = make_float2(-d[nt][2], -d[nt][3]);
    }
  }
  named_sync(bar_base, 128);
}

}  // namespace pf

using namespace pf;

// kLimbs = 1: the state enters the H-dependent MMA as one bf16 copy; 2: as
// two bf16 limbs hi + lo (page "ssm_gdn_tc_route.rs": the _tcfuse spine uses
// one limb of S_c, the _tcfuse_x2 spine two), the low limb staged in shared
// memory.
template <int kLimbs, bool kSeg>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                   const Params p) {
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned start, kept as an offset from the __shared__ array so
  // that accesses through it stay shared-space (not generic) loads and stores
  uint8_t* smem = smem_raw + ((uint32_t(1024) - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sbase = smem_u32(smem);
  const bool spine = int(blockIdx.x) < p.S;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (spine ? S_BARS : P_BARS));
  uint32_t* misc = reinterpret_cast<uint32_t*>(bars + 32);
  uint32_t* tmem_slot = misc;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
  int* sJ = reinterpret_cast<int*>(misc + 4);  // chunks per spine (preps only)
  volatile uint32_t* gabort = p.flags;
  uint32_t* err = &g_err_prefill;

  const int warp = int(warp_id_sync());
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int D = p.D;
  const int nbox = D / 64;
  const int units = p.num_seqs * p.H_v;
  const int vpg = p.H_v / p.H_k;

  for (uint32_t i = tid * 16; i < kSmemBytes; i += kThreads * 16)
    *reinterpret_cast<uint4*>(smem + i) = make_uint4(0, 0, 0, 0);
  __syncthreads();
  if (spine && tid < C) {  // the identity's diagonal (bf16 1.0), for the tensor cores
    *reinterpret_cast<uint16_t*>(smem + S_ID + sw128_offset(uint32_t(tid), uint32_t(2 * tid))) = 0x3F80u;
    fence_proxy_async_smem();
  }
  if (tid == 0) {
    if (spine) {
      for (int b = 0; b < SB_COUNT; ++b) mbar_init(&bars[b], 1u);
    } else {
      for (int b = 0; b < PB_COUNT; ++b) {
        uint32_t cnt = 1;
        if ((b >= PB_P1FREE && b < PB_P1FREE + 4) || b == PB_TREADY || b == PB_TREADY + 1) cnt = 128;
        if (b >= PB_GATEF && b < PB_GATEF + 4) cnt = 32;
        mbar_init(&bars[b], cnt);
      }
    }
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    if (spine && p.o != nullptr) tma_prefetch_desc(&tm_o);
  }
  // Chunks per spine, for the preps' item walk.
  int Jmax = 0;
  if (!spine) {
    for (int s = tid; s < p.S; s += kThreads) {
      int J = 0;
      for (int u = s; u < units; u += p.S) J += unit_chunks<kSeg>(p, u);
      sJ[s] = J;
    }
  }
  if (warp == 0) tmem_alloc(tmem_slot, 512);
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int ksteps_d = D / 16;
  if (!spine)
    for (int s = 0; s < p.S; ++s) Jmax = max(Jmax, sJ[s]);
  const int iend = Jmax * p.S;  // items i < iend (some invalid: chunk j beyond its spine)
  // Warps 0-7 (the spine's state warps, the preps' item groups) hold the
  // large register sets; the single-thread roles and the output warps give
  // theirs up: each role branch below starts with its warpgroup's change
  // (every warp of a warpgroup makes the same one).

  if (spine) {
    // =====================================================================
    // SPINE s = blockIdx.x
    // =====================================================================
    const int s = int(blockIdx.x);
    if (warp < 8) {
      setmaxnreg_inc<kRegsWide>();
      // ---------------- state warps: warp w serves TMEM lane quadrant w & 3
      // (row j of H^T) and half hh = w >> 2: columns d_k 64 hh .. 64 hh + 63 of
      // H^T (kept in registers, f32) and chunk rows 32 hh .. 32 hh + 31 of Vn^T
      // and of the outputs.  Per chunk c:
      //   H <- e^{G_C} H + dH (dH of chunk c-1, from TMEM); H^T in bf16 -> TMEM;
      //   [Vn | -O1]^T = [U^T I | 0] - H^T [W; Q]^T: one N = 128 MMA with B
      //   negated, accumulated onto U^T I (issued before the barrier, off
      //   this chain) and onto the zeros the output warps left;
      //   Vn^T, e^{G_C - G_r} Vn^T in bf16 -> TMEM, in place;
      //   dH^T = Vns^T K (A from TMEM); then, off this chain, O2^T = Vn^T Aqk^T;
      // warp 9 issues the MMAs right after the two named barriers; the
      // outputs are the output warps' (12 - 15), off this chain.
      const int qd = warp & 3, hh = warp >> 2;
      const int j = 32 * qd + lane;
      const uint32_t lane_off = uint32_t(32 * qd) << 16;
      const bool jv = j < D;
      float* eg_s = reinterpret_cast<float*>(smem + S_EG);
      float* ecg_s = reinterpret_cast<float*>(smem + S_ECG);
      // Every exit from these loops follows a bar.red agreement that the
      // issuer warp takes part in, so the two sides always leave together.
      int c = 0;
      bool ok = true;
      for (int u = s; u < units; u += p.S) {
        const int n = u / p.H_v, h = u % p.H_v;
        int tb, te;
        seq_range<kSeg>(p, n, tb, te);
        const size_t seq_off = size_t(n) * p.H_v * size_t(D) * D, head_off = size_t(h) * D * D;
        const float* h0b = (kSeg && p.h0_tab != nullptr) ? p.h0_tab[n]
                                               : (p.h0 != nullptr ? p.h0 + seq_off : nullptr);
        float* hTb = (kSeg && p.hT_tab != nullptr) ? p.hT_tab[n] : (p.hT != nullptr ? p.hT + seq_off : nullptr);
        bool agreed = true;
        float H[64];
        {
          const float* h0 = (h0b != nullptr && jv) ? h0b + head_off + j : nullptr;
#pragma unroll
          for (int i = 0; i < 64; ++i)
            H[i] = (h0 != nullptr && 64 * hh + i < D) ? h0[size_t(64 * hh + i) * D] : 0.f;
          if (kSeg && p.h0_identity) {
#pragma unroll
            for (int i = 0; i < 64; ++i) H[i] = (64 * hh + i == j) ? 1.f : 0.f;
          }
        }
        const int c_first = c;
        float dec_prev = 1.f;
        for (int t0 = tb; t0 < te; t0 += C, ++c) {
          const int st = c & 1;
          const float* sg = reinterpret_cast<const float*>(smem + S_STG + st * STG_BYTES + STG_GATE);
          if (c > c_first) {  // dH of the previous chunk landed
            ok = mbar_wait(&bars[SB_DHFULL], (c - 1) & 1, abort_flag, err, 16u, p.spin_limit) && ok;
            tc_fence_after();
          }
          ok = ok && mbar_wait(&bars[SB_AF + st], (c >> 1) & 1, abort_flag, err, 16u, p.spin_limit);
          if (c > c_first) {  // H <- e^{G_C} H + dH
#pragma unroll
            for (int q2 = 0; q2 < 2; ++q2) {
              float d[32];
              tmem_ld32(tmem + lane_off + ST_DH + 64u * uint32_t(hh) + 32u * uint32_t(q2), d);
              tmem_ld_wait();
#pragma unroll
              for (int i = 0; i < 32; ++i) H[32 * q2 + i] = fmaf(dec_prev, H[32 * q2 + i], d[i]);
            }
          }
          const float dec_cur = sg[128];
          // part A is released after the [W; Q] MMA: keep the gate factors
          // (the output factor negated: the MMA forms -O1)
          if (tid < 64) eg_s[64 * (c & 3) + tid] = -(sg[tid] * p.scale);
          else if (tid < 128) ecg_s[64 * st + tid - 64] = sg[tid];
          {
            // bf16 H^T row j, d_k 64 hh .. + 63, as the A operand of the [W; Q]
            // MMA in tensor memory (the previous chunk's [W; Q] MMA, done
            // before VOFULL, was the last reader)
            uint32_t hp[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) hp[i] = pack_bf16x2(H[2 * i], H[2 * i + 1]);
            tmem_st32u(tmem + lane_off + ST_HT + 32u * uint32_t(hh), hp);
            tmem_st_wait();
          }
          if constexpr (kLimbs == 2) {
            // the previous chunk's [W; Q] MMA read the low limb before VOFULL
            st_row64_bf16_lo(sbase + S_VN + uint32_t(hh) * 16384, uint32_t(j), H);
            fence_proxy_async_smem();
          }
          tc_fence_before();
          if (!named_all(1, kSpineSync, ok)) {  // the issuer warp starts [W; Q]
            agreed = false;
            break;
          }
          // Vn^T (f32, chunk rows 32 hh .. + 31) -> bf16 Vn^T and
          // e^{G_C - G_r} Vn^T in its own 32 columns: the A operands of O2 and
          // dH, k-steps 2 hh and 2 hh + 1 (Vn at +0, +8; Vns at +16, +24)
          ok = mbar_wait(&bars[SB_VOFULL], c & 1, abort_flag, err, 16u, p.spin_limit) && ok;
          tc_fence_after();
          {
            const float* ecp = ecg_s + 64 * st + 32 * hh;
            const uint32_t vcol = tmem + lane_off + ST_VO + 128u * uint32_t(st) + 32u * uint32_t(hh);
            float vn[32];
            uint32_t pk[32];
            tmem_ld32(vcol, vn);
            tmem_ld_wait();
#pragma unroll
            for (int i4 = 0; i4 < 8; ++i4) {
              const float4 e = *reinterpret_cast<const float4*>(ecp + 4 * i4);
              pk[2 * i4] = pack_bf16x2(vn[4 * i4], vn[4 * i4 + 1]);
              pk[2 * i4 + 1] = pack_bf16x2(vn[4 * i4 + 2], vn[4 * i4 + 3]);
              pk[16 + 2 * i4] = pack_bf16x2(e.x * vn[4 * i4], e.y * vn[4 * i4 + 1]);
              pk[17 + 2 * i4] = pack_bf16x2(e.z * vn[4 * i4 + 2], e.w * vn[4 * i4 + 3]);
            }
            tmem_st32u(vcol, pk);
            tmem_st_wait();
          }
          tc_fence_before();
          if (!named_all(1, kSpineSync, ok)) {  // the issuer warp starts dH, O2
            agreed = false;
            break;
          }
          dec_prev = dec_cur;
        }
        if (!agreed) {
          ok = false;
          break;
        }
        if (te > tb) {  // the last chunk's update
          ok = mbar_wait(&bars[SB_DHFULL], (c - 1) & 1, abort_flag, err, 16u, p.spin_limit) && ok;
          tc_fence_after();
#pragma unroll
          for (int q2 = 0; q2 < 2; ++q2) {
            float d[32];
            tmem_ld32(tmem + lane_off + ST_DH + 64u * uint32_t(hh) + 32u * uint32_t(q2), d);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i) H[32 * q2 + i] = fmaf(dec_prev, H[32 * q2 + i], d[i]);
          }
          tc_fence_before();
          if (!named_all(1, kSpineSync, ok)) {  // the issuer warp takes part
            ok = false;
            break;
          }
        }
        if (hTb != nullptr && jv) {
          float* hT = hTb + head_off + j;
#pragma unroll
          for (int i = 0; i < 64; ++i)
            if (64 * hh + i < D) hT[size_t(64 * hh + i) * D] = H[i];
        }
        tc_fence_before();
      }
    } else {
      setmaxnreg_dec<kRegsNarrow>();
      if (warp == 9) {
      // ---------------- issuer: joins the state warps' two barriers per chunk
      // (bar.red: every participant gets the same outcome) and issues
      //   before the first:  Vn^T := U^T I, once the output warps have read
      //                      chunk c-2 out of this buffer and zeroed its O1
      //                      half (OEMPTY: its dH and O2 are done with the Vn
      //                      half too)
      //   after the first:   [Vn | -O1]^T += H^T (-[W; Q])^T  (N = 128)
      //   after the second:  dH^T = Vns^T K (fresh), committed on its own
      //                      (DHFULL: the chain goes on), then O2^T = Vn^T
      //                      Aqk^T into the one O2 buffer once the output
      //                      warps have read chunk c-1's (OEMPTY); OFULL
      //                      covers both
      // A tcgen05.mma costs about the same to issue at N = 64 as at N = 128,
      // and one thread issues everything, so the stream has few and wide
      // MMAs; the shared-memory descriptors are built once and offset per
      // k-step, and the k-step loops have compile-time trip counts.
      const bool leader = lane == 0;
      const uint64_t dsw = make_sdesc_sw128(0, 16, 1024);    // K-major operands
      const uint64_t dswk = make_sdesc_sw128(0, 8192, 1024);  // K as the MN-major B of dH
      auto walk = [&](auto ks_tag) {
        constexpr int KS = decltype(ks_tag)::value;  // k-steps over d_k
        constexpr uint32_t id_dh = make_idesc_bf16(128, 128, 0, 1);
        constexpr uint32_t id_n64 = make_idesc_bf16(128, 64, 0, 0);
        constexpr uint32_t id_wq = make_idesc_bf16(128, 128, 0, 0, 1);  // B negated
        int c = 0;
        for (int u = s; u < units; u += p.S) {
          int tb, te;
          seq_range<kSeg>(p, u / p.H_v, tb, te);
          for (int t0 = tb; t0 < te; t0 += C, ++c) {
            const int st = c & 1;
            const uint32_t stg4 = (sbase + S_STG + uint32_t(st) * STG_BYTES) >> 4;
            const uint32_t vo = tmem + ST_VO + 128u * uint32_t(st);       // Vn | O1 of this chunk
            bool okw = true;
            if (leader) {
              okw = mbar_wait(&bars[SB_OEMPTY + st], (c >> 1) & 1, abort_flag, err, 16u, p.spin_limit);
              okw = okw && mbar_wait(&bars[SB_BF + st], (c >> 1) & 1, abort_flag, err, 16u, p.spin_limit);
              if (okw) {
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                  mma_bf16_ss(vo, dsw + (stg4 + (STG_U >> 4) + 2 * kk),
                              dsw + ((sbase + S_ID) >> 4) + 2 * kk, id_n64, kk > 0);
              }
            }
            okw = __shfl_sync(0xffffffffu, okw, 0);
            if (!named_all(1, kSpineSync, okw)) return false;
            if (leader) {
              tc_fence_after();
#pragma unroll
              for (int kk = 0; kk < KS; ++kk) {
                const uint32_t off4 = ((kk >> 2) * 16384 + (kk & 3) * 32) >> 4;
                mma_bf16_ts(vo, tmem + ST_HT + 8u * kk, dsw + (stg4 + (STG_WQ >> 4) + off4), id_wq, 1u);
                if constexpr (kLimbs == 2)
                  mma_bf16_ss(vo, dsw + (((sbase + S_VN) >> 4) + off4), dsw + (stg4 + (STG_WQ >> 4) + off4),
                              id_wq, 1u);
              }
              mma_commit(&bars[SB_VOFULL]);
              mma_commit(&bars[SB_AE + st]);
            }
            __syncwarp();
            if (!named_all(1, kSpineSync, true)) return false;
            if (leader) {
              tc_fence_after();
              // k-step kk: chunk rows 16 kk .. + 15, written by the state
              // warps of half kk >> 1 at column 32 (kk >> 1) + 8 (kk & 1)
              // (Vn), + 16 (Vns)
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                mma_bf16_ts(tmem + ST_DH, vo + 32u * uint32_t(kk >> 1) + 16u + 8u * uint32_t(kk & 1),
                            dswk + (stg4 + (STG_K >> 4) + 128 * kk), id_dh, kk > 0);
              mma_commit(&bars[SB_DHFULL]);
              if (c > 0)  // chunk c-1's O2 read out
                mbar_wait(&bars[SB_OEMPTY + (st ^ 1)], (((c - 1) >> 1) + 1) & 1, abort_flag, err, 16u,
                          p.spin_limit);
              tc_fence_after();
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                mma_bf16_ts(tmem + ST_O2, vo + 32u * uint32_t(kk >> 1) + 8u * uint32_t(kk & 1),
                            dsw + (stg4 + (STG_AQK >> 4) + 2 * kk), id_n64, kk > 0);
              mma_commit(&bars[SB_OFULL + st]);
              mma_commit(&bars[SB_BE + st]);
            }
            __syncwarp();
          }
          if (te > tb && !named_all(1, kSpineSync, true)) return false;  // the unit-end agreement
        }
        return true;
      };
      if (D == 128) walk(std::integral_constant<int, 8>{});
      else walk(std::integral_constant<int, 4>{});
      if (leader) {  // every MMA this thread issued has completed
        mma_commit(&bars[SB_DRAIN]);
        mbar_wait(&bars[SB_DRAIN], 0, nullptr, err, 8u);
      }
      __syncwarp();
      } else if (warp == 8) {
      // ---------------- feeder: chunk c into stage c & 1, part by part.
      // Part A (Q by TMA; W and the gates from the ring entry) as soon as
      // chunk c - 2's [W; Q] MMA is done; part B (K by TMA; U^T and Aqk)
      // once chunk c - 2's dH and O2 are done, when its ring entry also goes
      // back to the preps (before this chunk's entry is awaited).
      if (lane == 0) {
        ChunkIter fd;
        it_start<kSeg>(fd, p, s);
        int issued_a = 0, issued_b = 0;
        bool ok = true;
        while (fd.ok && ok) {
          const int cc = fd.c, st = cc & 1;
          uint8_t* stg = smem + S_STG + st * STG_BYTES;
          const int hk = fd.h / vpg;
          const uint8_t* src = ring_entry(p, s, cc % kRing);
          // ---- part A
          if (cc >= 2) {
            ok = mbar_wait(&bars[SB_AE + st], ((cc >> 1) & 1) ^ 1, abort_flag, err, 1u, p.spin_limit);
            if (!ok) break;
          }
          uint64_t* fa = &bars[SB_AF + st];
          // The phase completes on the one arrival (made with the ring bytes, or
          // bare on an abort) plus every byte announced before it.
          mbar_expect_tx(fa, uint32_t(nbox) * 8192);
          for (int b = 0; b < nbox; ++b)
            tma_load_3d(stg + STG_WQ + b * 16384 + 8192, &tm_q, fa, b * 64, hk, fd.t0);
          issued_a = cc + 1;
          // chunk cc - 2 fully consumed (its dH and O2 done): its ring entry
          // goes back to the preps before this chunk's is awaited
          if (cc >= 2) {
            ok = mbar_wait(&bars[SB_BE + st], ((cc >> 1) & 1) ^ 1, abort_flag, err, 1u, p.spin_limit);
            if (ok) st_release_gpu(free_flag(p, s, (cc - 2) % kRing), uint32_t(cc - 1));
          }
          ok = ok && poll_geq(ready_flag(p, s, cc % kRing), uint32_t(cc + 1), gabort, err, 1u, p.spin_limit);
          if (!ok) {  // the phase still completes once the Q tiles landed
            mbar_arrive(fa);
            break;
          }
          fence_proxy_async_global();
          mbar_arrive_expect_tx(fa, 2 * 8192 + G_GATE_BYTES);
          bulk_load_g2s(stg + STG_WQ, src + G_W, 8192, fa);
          bulk_load_g2s(stg + STG_WQ + 16384, src + G_W + 8192, 8192, fa);
          bulk_load_g2s(stg + STG_GATE, src + G_GATE, G_GATE_BYTES, fa);
          // ---- part B (its buffers freed with BE above)
          uint64_t* fb = &bars[SB_BF + st];
          mbar_arrive_expect_tx(fb, uint32_t(nbox) * 8192 + 16384 + 8192);
          for (int b = 0; b < nbox; ++b)
            tma_load_3d(stg + STG_K + b * 8192, &tm_k, fb, b * 64, hk, fd.t0);
          bulk_load_g2s(stg + STG_U, src + G_U, 16384, fb);
          bulk_load_g2s(stg + STG_AQK, src + G_AQK, 8192, fb);
          issued_b = cc + 1;
          it_next<kSeg>(fd, p);
        }
        if (!ok) {
          *abort_flag = 1;
          atomicExch(const_cast<uint32_t*>(gabort), 1u);
        }
        // nothing may still be landing in shared memory at exit
        for (int cc = issued_a - 2; cc < issued_a; ++cc)
          if (cc >= 0) mbar_wait(&bars[SB_AF + (cc & 1)], (cc >> 1) & 1, nullptr, err, 32u);
        for (int cc = issued_b - 2; cc < issued_b; ++cc)
          if (cc >= 0) mbar_wait(&bars[SB_BF + (cc & 1)], (cc >> 1) & 1, nullptr, err, 32u);
      }
      __syncwarp();
      } else if (warp >= 12) {
        // ---------------- output warps, off the chain: for every chunk c of
        // this spine, once OFULL(c), warp 12 + q reads TMEM lane quadrant q
        // (d_v 32 q .. 32 q + 31) of -O1^T (upper half of the VO buffer) and
        // O2^T, 16 lanes x 16 chunk rows at a time in the 16x256b form, forms
        // o_r = scale e^{G_r} O1[r] + O2[r] in bf16 and writes it with
        // transposing matrix stores into the output tile of the chunk's
        // parity: two 64-column halves of [64 rows][128 B], 16-byte chunks
        // swizzled by row (the tensor stores' 128-byte swizzle).  Then it
        // zeroes the O1 half (the next [W; Q] MMA into this buffer
        // accumulates onto it), hands the TMEM buffers back to the issuer
        // (OEMPTY; both buffers once at start-up, zeroed), and one thread
        // stores the full 16-row blocks with TMA tensor stores; the rows of a
        // ragged block go out with plain stores.  A tile is rewritten two
        // chunks later, and the storing thread sees every earlier store
        // finish reading before the barrier that precedes that rewrite.
        const int qd = warp & 3;
        const int tq = lane & 3;                  // fragment column pair
        const int sm = lane >> 3, sk = lane & 7;  // stored matrix, stored row
        const float* eg_s = reinterpret_cast<const float*>(smem + S_EG);
        const bool elect = warp == 12 && lane == 0;
        const int halves = D / 64;
        const uint32_t zeros[32] = {};
        const uint32_t o1q = tmem + (uint32_t(32 * qd) << 16) + ST_VO + 64u;  // + 128 ob: O1 half
        for (int ob = 0; ob < 2; ++ob) {
          tmem_st32u(o1q + 128u * uint32_t(ob), zeros);
          tmem_st32u(o1q + 128u * uint32_t(ob) + 32u, zeros);
        }
        tmem_st_wait();
        tc_fence_before();
        named_sync(2, 128);
        if (elect) {
          mbar_arrive(&bars[SB_OEMPTY]);
          mbar_arrive(&bars[SB_OEMPTY + 1]);
        }
        int c = 0;
        bool ok = true;
        for (int u = s; u < units && ok; u += p.S) {
          const int h = u % p.H_v;
          int tb, te;
          seq_range<kSeg>(p, u / p.H_v, tb, te);
          for (int t0 = tb; t0 < te; t0 += C, ++c) {
            const int ob = c & 1, L = min(C, te - t0);
            bool okc =
                mbar_wait(&bars[SB_OFULL + ob], (c >> 1) & 1, abort_flag, err, 128u, p.spin_limit);
            tc_fence_after();
            const float* egp = eg_s + 64 * (c & 3);
            const uint32_t tile = S_OT + 16384u * uint32_t(ob);
#pragma unroll 1
            for (int r0 = 0; r0 < 64; r0 += 16) {
              // both 16-lane halves of the quadrant: four loads, one wait
              float a1[2][8], a2[2][8];
#pragma unroll
              for (int hf = 0; hf < 2; ++hf) {
                const uint32_t lb = uint32_t(32 * qd + 16 * hf);  // TMEM lane base (d_v)
                if (int(lb) < D) {  // warp-uniform (d = 64: quadrants 2, 3 empty)
                  tmem_ld_16x256b_x2(tmem + (lb << 16) + ST_VO + 128u * uint32_t(ob) + 64u + uint32_t(r0), a1[hf]);
                  tmem_ld_16x256b_x2(tmem + (lb << 16) + ST_O2 + uint32_t(r0), a2[hf]);
                }
              }
              tmem_ld_wait();
              const float2 e0 = *reinterpret_cast<const float2*>(egp + r0 + 2 * tq);
              const float2 e1 = *reinterpret_cast<const float2*>(egp + r0 + 8 + 2 * tq);
#pragma unroll
              for (int hf = 0; hf < 2; ++hf) {
                const int lb = 32 * qd + 16 * hf;
                if (lb >= D) continue;
                // fragments: rows = d_v lb + t / 4 (+ 8), columns = chunk rows
                // r0 + 2 (t % 4), + 1 (+ 8)
                const float* x = a1[hf];
                const float* y = a2[hf];
                const uint32_t m0 = pack_bf16x2(fmaf(e0.x, x[0], y[0]), fmaf(e0.y, x[1], y[1]));
                const uint32_t m1 = pack_bf16x2(fmaf(e0.x, x[2], y[2]), fmaf(e0.y, x[3], y[3]));
                const uint32_t m2 = pack_bf16x2(fmaf(e1.x, x[4], y[4]), fmaf(e1.y, x[5], y[5]));
                const uint32_t m3 = pack_bf16x2(fmaf(e1.x, x[6], y[6]), fmaf(e1.y, x[7], y[7]));
                // stored row sk of matrix sm: chunk row r0 + sk (+ 8), d_v lb (+ 8)
                const int row = r0 + sk + 8 * (sm >> 1);
                const int c0 = lb + 8 * (sm & 1);
                const uint32_t addr = sbase + tile + uint32_t(c0 >> 6) * 8192u + uint32_t(row) * 128u +
                                      (uint32_t(((c0 & 63) >> 3) ^ (row & 7)) << 4);
                if (okc) stmatrix_x4_trans(addr, m0, m1, m2, m3);
              }
            }
            tmem_st32u(o1q + 128u * uint32_t(ob), zeros);
            tmem_st32u(o1q + 128u * uint32_t(ob) + 32u, zeros);
            tmem_st_wait();
            tc_fence_before();
            fence_proxy_async_smem();  // the tile, before the tensor stores read it
            if (elect) tma_store_wait_read<0>();  // the other tile's stores (chunk c - 1)
            if (!named_all(2, 128, okc)) {
              ok = false;
              break;
            }
            if (elect) {
              mbar_arrive(&bars[SB_OEMPTY + ob]);
              if (p.o != nullptr) {
                for (int r0 = 0; r0 + 16 <= L; r0 += 16)
                  for (int hf = 0; hf < halves; ++hf)
                    tma_store_3d(&tm_o, smem + tile + uint32_t(hf) * 8192u + uint32_t(r0) * 128u, 64 * hf,
                                 h, t0 + r0);
                tma_store_commit();
              }
            }
            if ((L & 15) != 0 && p.o != nullptr) {  // rows L & ~15 .. L - 1: 16-byte pieces
              const int rb = L & ~15, per_row = D / 8, t = 32 * qd + lane;
              for (int id = t; id < (L - rb) * per_row; id += 128) {
                const int i = id / per_row, sg = id - i * per_row, row = rb + i;
                *reinterpret_cast<uint4*>(p.o + (size_t(t0 + row) * p.H_v + h) * D + 8 * sg) =
                    ld_shared_v4(sbase + tile + uint32_t(sg >> 3) * 8192u + uint32_t(row) * 128u +
                                 (uint32_t((sg & 7) ^ (row & 7)) << 4));
              }
            }
          }
        }
        if (elect) tma_store_wait_all<0>();  // every output store is complete
        __syncwarp();
      }  // warps 10 and 11: no spine role
    }
  } else {
    // =====================================================================
    // PREP prank = blockIdx.x - S: items k = 0, 1, ... of this CTA in order.
    // Item k: group g = k & 1 (warps 4g .. 4g+3), kg = k >> 1 its index in the
    // group, tile set k % 3, P1 TMEM buffer and gate block kg & 1 of group g.
    // =====================================================================
    const int prank = int(blockIdx.x) - p.S;
    if (warp < 8) {
      setmaxnreg_inc<kRegsWide>();
      // ---------------- groups: 128 threads each, items k = g, g + 2, ...
      const int g = warp >> 2;
      const int pt = tid & 127;
      const uint32_t lane_off = uint32_t((warp & 3) * 32) << 16;
      uint8_t* ga = smem + P_GRP + g * P_GS;
      float* M = reinterpret_cast<float*>(ga + GA_AF);
      float* Xs = reinterpret_cast<float*>(ga + GA_XS);
      const int gbar = 1 + 3 * g;  // this group's named barriers: gbar (all), gbar+1, gbar+2
      PrepIter it;
      pi_start<kSeg>(it, p, sJ, iend, prank);
      pi_align<kSeg>(it, p, sJ, iend, g);
      while (it.ok) {
        const int k = it.k, kg = k >> 1, t = k % 3, pb = kg & 1;
        uint8_t* set = smem + t * P_SET;
        const float* gt = reinterpret_cast<const float*>(ga + GA_GT + pb * PG_BYTES);
        const uint32_t tm = tmem + PT_WG * g;
        // gates written, P1 done (the group's Aqk buffer was copied into the
        // set of its previous item k - 2 at that item's end)
        const bool ready =
            mbar_wait(&bars[PB_GATEF + 2 * g + pb], (kg >> 1) & 1, abort_flag, err, 4u, p.spin_limit) &&
            mbar_wait(&bars[PB_P1F + 2 * g + pb], (kg >> 1) & 1, abort_flag, err, 4u, p.spin_limit);
        if (!named_all(gbar, 128, ready)) break;
        tc_fence_after();
        // ---- P1 row pt: K K^T (pt < 64) or Q K^T (pt >= 64), times e^{G_r - G_s}
        // (s <= r): two factors <= 1 for the blocks of s before r's 16-row
        // block, a direct exponential inside it.  One 16-column block per
        // pass of a loop kept rolled: the two 16-row halves of a warp take
        // different branches, and unrolled code this size runs from a cold
        // instruction cache.
        {
          const int r = pt & 63, rb = r >> 4;
          const float Gr = gt[PG_G + r];
          const float e1 = gt[PG_E1 + r];
          const float rf = pt < 64 ? gt[PG_BET + r] : p.scale;
          const float* e2 = gt + PG_E2 + 64 * rb;
#pragma unroll 1
          for (int sb = 0; sb < 4; ++sb) {
            float v[16], f[16];
            tmem_ld16(tm + lane_off + 64u * pb + 16u * uint32_t(sb), v);
            tmem_ld_wait();
            if (sb == 3) {
              tc_fence_before();
              mbar_arrive(&bars[PB_P1FREE + 2 * g + pb]);
            }
            const int s0 = 16 * sb;
            // strict lower triangle for A, lower triangle with the diagonal for Aqk
            const int lim = pt < 64 ? r - s0 - 1 : r - s0;
            if (sb < rb) {
#pragma unroll
              for (int jj = 0; jj < 16; jj += 4) {
                const float4 e4 = *reinterpret_cast<const float4*>(e2 + s0 + jj);
                f[jj] = rf * e1 * e4.x;
                f[jj + 1] = rf * e1 * e4.y;
                f[jj + 2] = rf * e1 * e4.z;
                f[jj + 3] = rf * e1 * e4.w;
              }
            } else if (sb == rb) {  // the row's own block: one exponential each
#pragma unroll
              for (int jj = 0; jj < 16; jj += 4) {
                const float4 g4 = *reinterpret_cast<const float4*>(gt + PG_G + s0 + jj);
                f[jj] = jj <= lim ? rf * __expf(Gr - g4.x) : 0.f;
                f[jj + 1] = jj + 1 <= lim ? rf * __expf(Gr - g4.y) : 0.f;
                f[jj + 2] = jj + 2 <= lim ? rf * __expf(Gr - g4.z) : 0.f;
                f[jj + 3] = jj + 3 <= lim ? rf * __expf(Gr - g4.w) : 0.f;
              }
            } else {  // above the diagonal block: zeros, no exponentials
#pragma unroll
              for (int jj = 0; jj < 16; ++jj) f[jj] = 0.f;
            }
            if (pt < 64) {  // A[r][s] = beta_r e^{G_r-G_s} k_r.k_s, s < r
#pragma unroll
              for (int jj = 0; jj < 16; jj += 4)
                *reinterpret_cast<float4*>(M + r * kAS + s0 + jj) =
                    make_float4(f[jj] * v[jj], f[jj + 1] * v[jj + 1], f[jj + 2] * v[jj + 2],
                                f[jj + 3] * v[jj + 3]);
            } else {  // Aqk[r][s] = scale e^{G_r-G_s} q_r.k_s, s <= r  (bf16, swizzled)
#pragma unroll
              for (int hc = 0; hc < 2; ++hc) {
                const int o = 8 * hc;
                *reinterpret_cast<uint4*>(ga + GA_AQK + sw128_offset(r, (2 * sb + hc) * 16)) =
                    make_uint4(pack_bf16x2(f[o] * v[o], f[o + 1] * v[o + 1]),
                               pack_bf16x2(f[o + 2] * v[o + 2], f[o + 3] * v[o + 3]),
                               pack_bf16x2(f[o + 4] * v[o + 4], f[o + 5] * v[o + 5]),
                               pack_bf16x2(f[o + 6] * v[o + 6], f[o + 7] * v[o + 7]));
              }
            }
          }
        }
        named_sync(gbar, 128);
        // ---- T = (I + A)^{-1}, in place
        invert_unit_lower64(M, Xs, pt, gbar);
        // ---- T1 = T diag(beta e^G) (rows pt < 64), T2 = T diag(beta) (rows pt >= 64),
        // into the item's Q boxes (Q was last read by P1)
        {
          const int r = pt & 63;
          const float* scv = gt + (pt < 64 ? PG_BEG : PG_BET);
          uint8_t* tile = set + (pt < 64 ? P_T1B : P_T2B);
#pragma unroll 1
          for (int cc = 0; cc < 8; ++cc) {
            const float4 ta = *reinterpret_cast<const float4*>(M + r * kAS + 8 * cc);
            const float4 tb2 = *reinterpret_cast<const float4*>(M + r * kAS + 8 * cc + 4);
            const float4 sa = *reinterpret_cast<const float4*>(scv + 8 * cc);
            const float4 sb2 = *reinterpret_cast<const float4*>(scv + 8 * cc + 4);
            const int s0 = 8 * cc;
            *reinterpret_cast<uint4*>(tile + sw128_offset(r, cc * 16)) = make_uint4(
                pack_bf16x2(s0 + 0 <= r ? ta.x * sa.x : 0.f, s0 + 1 <= r ? ta.y * sa.y : 0.f),
                pack_bf16x2(s0 + 2 <= r ? ta.z * sa.z : 0.f, s0 + 3 <= r ? ta.w * sa.w : 0.f),
                pack_bf16x2(s0 + 4 <= r ? tb2.x * sb2.x : 0.f, s0 + 5 <= r ? tb2.y * sb2.y : 0.f),
                pack_bf16x2(s0 + 6 <= r ? tb2.z * sb2.z : 0.f, s0 + 7 <= r ? tb2.w * sb2.w : 0.f));
          }
        }
        fence_proxy_async_smem();
        mbar_arrive(&bars[PB_TREADY + g]);
        // ---- W (row-major), U^T into [0, 32 KB) of the item's set
        if (!named_all(gbar, 128, mbar_wait(&bars[PB_WUF + g], kg & 1, abort_flag, err, 4u, p.spin_limit))) break;
        tc_fence_after();
        {
          // U^T: TMEM lane pt is row pt of U^T, stored as it is.  W: TMEM lane
          // pt is d_k column pt of W; 16 lanes x 16 chunk rows at a time in
          // the 16x256b form, then transposing matrix stores write whole
          // 16-byte row pieces of row-major W into its two 128B-swizzled boxes.
          const int wq = warp & 3, sm = lane >> 3, sk = lane & 7;
          const uint32_t wbase = smem_u32(set) + G_W;
#pragma unroll 1
          for (int hf = 0; hf < 2; ++hf) {
            float uv[32], wf[4][8];
            tmem_ld32(tm + lane_off + PT_U + 32u * hf, uv);
#pragma unroll
            for (int b4 = 0; b4 < 4; ++b4) {  // (lane half, 16-row block)
              const uint32_t lb = uint32_t(32 * wq + 16 * (b4 & 1));
              tmem_ld_16x256b_x2(tm + (lb << 16) + PT_W + 32u * hf + 16u * uint32_t(b4 >> 1), wf[b4]);
            }
            tmem_ld_wait();
#pragma unroll
            for (int hc = 0; hc < 4; ++hc) {
              const uint32_t off = sw128_offset(pt, (4 * hf + hc) * 16);
              *reinterpret_cast<uint4*>(set + G_U + off) =
                  make_uint4(pack_bf16x2(uv[8 * hc], uv[8 * hc + 1]),
                             pack_bf16x2(uv[8 * hc + 2], uv[8 * hc + 3]),
                             pack_bf16x2(uv[8 * hc + 4], uv[8 * hc + 5]),
                             pack_bf16x2(uv[8 * hc + 6], uv[8 * hc + 7]));
            }
#pragma unroll
            for (int b4 = 0; b4 < 4; ++b4) {
              const float* x = wf[b4];
              const int dk = 32 * wq + 16 * (b4 & 1) + 8 * (sm & 1);
              const int row = 32 * hf + 16 * (b4 >> 1) + sk + 8 * (sm >> 1);
              stmatrix_x4_trans(wbase + uint32_t(dk >> 6) * 8192u + uint32_t(row) * 128u +
                                    (uint32_t(((dk & 63) >> 3) ^ (row & 7)) << 4),
                                pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]),
                                pack_bf16x2(x[4], x[5]), pack_bf16x2(x[6], x[7]));
            }
          }
          // Aqk into the set's V boxes (free once the U MMA is done), so that
          // the group's buffer is its own again for item k + 2
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const uint32_t off = uint32_t(pt) * 64u + uint32_t(q) * 16u;
            *reinterpret_cast<uint4*>(set + P_V + off) = *reinterpret_cast<const uint4*>(ga + GA_AQK + off);
          }
        }
        tc_fence_before();
        fence_proxy_async_smem();
        named_sync(gbar, 128);
        if (pt == 0) mbar_arrive(&bars[PB_STAGED + g]);
        pi_next<kSeg>(it, p, sJ, iend);
        pi_align<kSeg>(it, p, sJ, iend, g);
      }
    } else {
      setmaxnreg_dec<kRegsNarrow>();
      if (warp == 8) {
      // ---------------- loader: item k's K, Q, V tiles (TMA, lane 0) once set
      // k % 3 is free (item k - 3 stored)
      PrepIter it;
      pi_start<kSeg>(it, p, sJ, iend, prank);
      int last_k = -1;
      bool ok = true;
      while (it.ok && ok) {
        const int k = it.k, t = k % 3;
        ok = k < 3 || mbar_wait(&bars[PB_STORED + t], ((k / 3) & 1) ^ 1, abort_flag, err, 1u, p.spin_limit);
        if (!__all_sync(0xffffffffu, ok)) {
          ok = false;
          break;
        }
        if (lane == 0) {
          uint64_t* fb = &bars[PB_KQVF + t];
          mbar_arrive_expect_tx(fb, uint32_t(nbox) * ((kSeg && p.v_zero) ? 2 : 3) * 8192);
          uint8_t* set = smem + t * P_SET;
          const int hk = it.h / vpg;
          for (int b2 = 0; b2 < nbox; ++b2) {
            tma_load_3d(set + P_KQ + b2 * 16384, &tm_k, fb, b2 * 64, hk, it.t0);
            tma_load_3d(set + P_KQ + b2 * 16384 + 8192, &tm_q, fb, b2 * 64, hk, it.t0);
            // v read as zeros: the V boxes keep the zeros of the start-up clear
            if (!(kSeg && p.v_zero)) tma_load_3d(set + P_V + b2 * 8192, &tm_v, fb, b2 * 64, it.h, it.t0);
          }
          last_k = k;
        }
        pi_next<kSeg>(it, p, sJ, iend);
      }
      if (!ok) {
        *abort_flag = 1;
        atomicExch(const_cast<uint32_t*>(gabort), 1u);
      }
      if (lane == 0)  // nothing may still be landing in shared memory at exit
        for (int k = last_k - 2; k <= last_k; ++k)
          if (k >= 0) mbar_wait(&bars[PB_KQVF + k % 3], (k / 3) & 1, nullptr, err, 32u);
      __syncwarp();
    } else if (warp == 9) {
      // ---------------- MMA issue for both groups, whichever is ready: P1 of
      // items in order (tiles landed, the group's P1 buffer read back), W/U of
      // each group's next item once its T is ready
      if (elect_one()) {
        const uint32_t id_p1 = make_idesc_bf16(128, 64, 0, 0);
        const uint32_t id_wu = make_idesc_bf16(128, 64, 1, 0);
        PrepIter itp;
        pi_start<kSeg>(itp, p, sJ, iend, prank);
        int kp = 0;                // next item for P1
        int kw[2] = {0, 0};        // next in-group index for W/U
        long long last = clock64();
        while (true) {
          bool prog = false;
          if (itp.ok) {
            const int t = kp % 3, g = kp & 1, kg = kp >> 1, pb = kg & 1;
            if (mbar_test_wait(&bars[PB_KQVF + t], (kp / 3) & 1) &&
                (kg < 2 || mbar_test_wait(&bars[PB_P1FREE + 2 * g + pb], ((kg >> 1) & 1) ^ 1))) {
              tc_fence_after();
              const uint32_t set = sbase + t * P_SET;
              const uint32_t tm = tmem + PT_WG * g + 64u * pb;
              for (int kk = 0; kk < ksteps_d; ++kk) {
                const uint32_t a = set + P_KQ + (kk >> 2) * 16384 + (kk & 3) * 32;
                mma_bf16_ss(tm, make_sdesc_sw128(a, 16, 1024), make_sdesc_sw128(a, 16, 1024), id_p1,
                            kk > 0);
              }
              mma_commit(&bars[PB_P1F + 2 * g + pb]);
              ++kp;
              pi_next<kSeg>(itp, p, sJ, iend);
              prog = true;
            }
          }
#pragma unroll
          for (int g = 0; g < 2; ++g) {
            const int kwg = kw[g], k = 2 * kwg + g;
            if (k < kp && mbar_test_wait(&bars[PB_TREADY + g], kwg & 1)) {
              tc_fence_after();
              const uint32_t set = sbase + (k % 3) * P_SET;
              const uint32_t tm = tmem + PT_WG * g;
              for (int kk = 0; kk < 4; ++kk)
                mma_bf16_ss(tm + PT_W, make_sdesc_sw128(set + P_KQ + kk * 2048, 16384, 1024),
                            make_sdesc_sw128(set + P_T1B + kk * 32, 16, 1024), id_wu, kk > 0);
              for (int kk = 0; kk < 4; ++kk)
                mma_bf16_ss(tm + PT_U, make_sdesc_sw128(set + P_V + kk * 2048, 8192, 1024),
                            make_sdesc_sw128(set + P_T2B + kk * 32, 16, 1024), id_wu, kk > 0);
              mma_commit(&bars[PB_WUF + g]);
              ++kw[g];
              prog = true;
            }
          }
          if ((!itp.ok && 2 * kw[0] >= kp && 2 * kw[1] + 1 >= kp) || *abort_flag) break;
          if (prog) {
            last = clock64();
          } else {
            if (clock64() - last > p.spin_limit) {
              *abort_flag = 1;
              atomicExch(const_cast<uint32_t*>(gabort), 1u);
              atomicOr(err, 2u);
              break;
            }
            __nanosleep(32);
          }
        }
        mma_commit(&bars[PB_DRAIN]);
        mbar_wait(&bars[PB_DRAIN], 0, nullptr, err, 8u);
      }
      __syncwarp();
    } else if (warp == 10) {
      // ---------------- store: each staged item to its spine's ring entry, in
      // item order
      if (lane == 0) {
        PrepIter it;
        pi_start<kSeg>(it, p, sJ, iend, prank);
        bool ok = true;
        while (it.ok && ok) {
          const int k = it.k, t = k % 3, g = k & 1, kg = k >> 1;
          const int e = it.j % kRing;
          ok = mbar_wait(&bars[PB_STAGED + g], kg & 1, abort_flag, err, 4u, p.spin_limit);
          if (ok && it.j >= kRing)  // entry e is free once the spine copied item j - kRing
            ok = poll_geq(free_flag(p, it.s, e), uint32_t(it.j - kRing + 1), gabort, err, 4u, p.spin_limit);
          if (!ok) break;
          fence_proxy_async_global();
          uint8_t* dst = ring_entry(p, it.s, e);
          const uint8_t* ga = smem + P_GRP + g * P_GS;
          // W | U^T | Aqk: the set's first 40 KB, laid out as the ring entry
          bulk_store_s2g(dst + G_W, smem + t * P_SET, 40960);
          bulk_store_s2g(dst + G_GATE, ga + GA_GT + (kg & 1) * PG_BYTES + PG_EG * 4, G_GATE_BYTES);
          tma_store_commit();
          tma_store_wait_read<0>();
          mbar_arrive(&bars[PB_STORED + t]);
          mbar_arrive(&bars[PB_GBFREE + 2 * g + (kg & 1)]);
          tma_store_wait_all<0>();
          fence_proxy_async_global();
          st_release_gpu(ready_flag(p, it.s, e), uint32_t(it.j + 1));
          pi_next<kSeg>(it, p, sJ, iend);
        }
        if (!ok) {
          *abort_flag = 1;
          atomicExch(const_cast<uint32_t*>(gabort), 1u);
        }
      }
      __syncwarp();
    } else if (warp == 11) {
      // ---------------- gate factors of item k (whole warp), into gate block
      // kg & 1 of group k & 1 once the store of item k - 4, the block's last
      // reader, has read it (GBFREE), beside the loader
      PrepIter it;
      pi_start<kSeg>(it, p, sJ, iend, prank);
      bool ok = true;
      while (it.ok && ok) {
        const int k = it.k, g = k & 1, gb = (k >> 1) & 1;
        ok = k < 4 || mbar_wait(&bars[PB_GBFREE + 2 * g + gb], ((k >> 2) & 1) ^ 1, abort_flag, err, 1u,
                                p.spin_limit);
        if (!__all_sync(0xffffffffu, ok)) {
          ok = false;
          break;
        }
        // padded rows: g = beta = 0; lane l owns rows 2l, 2l + 1
        float* gt = reinterpret_cast<float*>(smem + P_GRP + g * P_GS + GA_GT + gb * PG_BYTES);
        {
          const int r0 = 2 * lane;
          const float* gsrc = p.g + size_t(it.t0) * p.gb_stride + it.h;
          const float* bsrc = p.beta + size_t(it.t0) * p.gb_stride + it.h;
          const float a0 = r0 < it.L ? gsrc[size_t(r0) * p.gb_stride] : 0.f;
          const float a1 = r0 + 1 < it.L ? gsrc[size_t(r0 + 1) * p.gb_stride] : 0.f;
          const float b0 = r0 < it.L ? bsrc[size_t(r0) * p.gb_stride] : 0.f;
          const float b1 = r0 + 1 < it.L ? bsrc[size_t(r0 + 1) * p.gb_stride] : 0.f;
          float s2 = a0 + a1;
#pragma unroll
          for (int off = 1; off < 32; off <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, s2, off);
            if (lane >= off) s2 += y;
          }
          const float G1 = s2, G0 = s2 - a1;       // G_{r0+1}, G_{r0}
          const float GC = __shfl_sync(0xffffffffu, G1, 31);
          {
            // Every decay factor is e^{G_r - G_s} for some s <= r (G_{-1} = 0):
            // finite while the gates rise by at most kGateRise after any row
            // of the chunk.  A larger rise (positive gates) is flagged.
            float mn = fminf(fminf(G0, G1), 0.f);
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
              const float y = __shfl_up_sync(0xffffffffu, mn, off);
              if (lane >= off) mn = fminf(mn, y);
            }
            float before = __shfl_up_sync(0xffffffffu, mn, 1);  // min over rows < r0
            if (lane == 0) before = 0.f;
            const float m0 = fminf(before, G0), m1 = fminf(m0, G1);
            float rise = fmaxf(G0 - m0, G1 - m1);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1)
              rise = fmaxf(rise, __shfl_xor_sync(0xffffffffu, rise, off));
            if (lane == 0 && !(rise <= kGateRise)) atomicOr(err, kErrGateRise);
          }
          // G at the start of this pair's 16-row block: row r0 & ~15 is the
          // first row of lane (r0 & ~15) / 2
          const float Gb = __shfl_sync(0xffffffffu, G0, (r0 & ~15) >> 1);
          gt[PG_G + r0] = G0;
          gt[PG_G + r0 + 1] = G1;
          gt[PG_BET + r0] = b0;
          gt[PG_BET + r0 + 1] = b1;
          const float eg0 = __expf(G0), eg1 = __expf(G1);
          gt[PG_EG + r0] = eg0;
          gt[PG_EG + r0 + 1] = eg1;
          gt[PG_BEG + r0] = b0 * eg0;
          gt[PG_BEG + r0 + 1] = b1 * eg1;
          gt[PG_ECG + r0] = __expf(GC - G0);
          gt[PG_ECG + r0 + 1] = __expf(GC - G1);
          gt[PG_E1 + r0] = __expf(G0 - Gb);
          gt[PG_E1 + r0 + 1] = __expf(G1 - Gb);
          if (lane == 0) gt[PG_DEC] = __expf(GC);
          __syncwarp();
          // E2[bb][s2] = e^{G_{16 bb} - G_s2}, s2 < 16 bb
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const int e2 = lane + 32 * q, bb = e2 >> 6, sx = e2 & 63;
            gt[PG_E2 + e2] = (sx < 16 * bb) ? __expf(gt[PG_G + 16 * bb] - gt[PG_G + sx]) : 0.f;
          }
        }
        mbar_arrive(&bars[PB_GATEF + 2 * g + gb]);  // release: this lane's gate writes
        pi_next<kSeg>(it, p, sJ, iend);
      }
      if (!ok) {
        *abort_flag = 1;
        atomicExch(const_cast<uint32_t*>(gabort), 1u);
      }
      __syncwarp();
      }  // warps 12 - 15: no prep role
    }
  }

  // ---- teardown: publish an abort to the grid, release TMEM
  tc_fence_before();
  __syncthreads();
  if (tid == 0 && *abort_flag) atomicExch(const_cast<uint32_t*>(gabort), 1u);
  if (warp == 0) tmem_dealloc(tmem, 512);
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------

namespace {

// CTAs of this kernel that can be resident at once on the current device.
int resident_ctas() {
  static int cache[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  int* slot = (dev >= 0 && dev < 64) ? &cache[dev] : nullptr;
  if (slot != nullptr && *slot > 0) return *slot;
  int per_sm = 0;
  cudaFuncSetAttribute(prefill_kernel<1, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       int(kSmemAlloc));
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, prefill_kernel<1, false>, kThreads,
                                                    kSmemAlloc) != cudaSuccess) {
    cudaGetLastError();
    per_sm = 0;
  }
  const int m = per_sm * sm_count();
  if (slot != nullptr && m > 0) *slot = m;
  return m;
}

// Grid and spine count for `units` (sequence, v-head) units: one CTA per SM,
// about a third of them spines (each prep serves two spines' worth of
// chunks), never more spines than units.
void plan(int units, int* grid, int* spines) {
  const int G = resident_ctas();
  *grid = G;
  int S = G / 3;
  if (S > units) S = units;
  if (S > kMaxSpines) S = kMaxSpines;
  if (S < 1) S = 1;
  *spines = S;
}

size_t flag_bytes(int S) { return (size_t(1 + S * kRing) * kFlagLine + 1023) / 1024 * 1024; }

}  // namespace

// Diagnostics only (gdn_debug_set_spin_limit): a shorter give-up time for the
// prefill's pipeline waits, so that a test can make them run out.
static long long g_spin_limit_override = 0;

void set_prefill_spin_limit(long long cycles) { g_spin_limit_override = cycles > 0 ? cycles : 0; }

size_t prefill_ring_bytes(int units) {
  int G = 0, S = 0;
  plan(units, &G, &S);
  return flag_bytes(S) + size_t(S) * kRing * SLOT_G;
}

int prefill_spine_budget() {
  int G = 0, S = 0;
  plan(1 << 20, &G, &S);
  return S;
}

cudaError_t launch_prefill_call(const PrefillCall& c, cudaStream_t s) {
  const int D = c.D;
  CUtensorMap tq, tk, tv;
  {
    uint64_t dims[3] = {uint64_t(D), uint64_t(c.H_k), uint64_t(c.total_tokens)};
    uint64_t strides[2] = {uint64_t(D) * 2, uint64_t(c.qk_stride) * 2};
    uint32_t box[3] = {64, 1, 64};
    if (!encode_tmap_bf16(&tq, c.q, 3, dims, strides, box, true)) return cudaErrorInvalidValue;
    if (!encode_tmap_bf16(&tk, c.k, 3, dims, strides, box, true)) return cudaErrorInvalidValue;
  }
  {
    uint64_t dims[3] = {uint64_t(D), uint64_t(c.H_v), uint64_t(c.total_tokens)};
    uint64_t strides[2] = {uint64_t(D) * 2, uint64_t(c.v_stride) * 2};
    uint32_t box[3] = {64, 1, 64};
    if (!encode_tmap_bf16(&tv, c.v, 3, dims, strides, box, true)) return cudaErrorInvalidValue;
  }
  // o [T, H_v, d_v]: the spines store 16 rows x 64 columns of one head at a time
  CUtensorMap to;
  memset(&to, 0, sizeof(to));
  if (c.o != nullptr) {
    uint64_t dims[3] = {uint64_t(D), uint64_t(c.H_v), uint64_t(c.total_tokens)};
    uint64_t strides[2] = {uint64_t(D) * 2, uint64_t(c.H_v) * uint64_t(D) * 2};
    uint32_t box[3] = {64, 1, 16};  // 16 rows x 64 columns, 128-byte swizzle
    if (!encode_tmap_bf16(&to, c.o, 3, dims, strides, box, true)) return cudaErrorInvalidValue;
  }
  // The plain form (whole sequences, h0 / hT arrays, real v) carries none of
  // the segment-pass branches.
  const bool seg = c.seg != nullptr || c.h0_tab != nullptr || c.hT_tab != nullptr || c.v_zero ||
                   c.h0_identity;
  auto kernel = c.limbs == 2 ? (seg ? prefill_kernel<2, true> : prefill_kernel<2, false>)
                             : (seg ? prefill_kernel<1, true> : prefill_kernel<1, false>);
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       int(kSmemAlloc));
  if (e != cudaSuccess) return e;
  int G = 0, S = 0;
  plan(c.num_seqs * c.H_v, &G, &S);
  if (G < 2) return cudaErrorCooperativeLaunchTooLarge;
  Params p;
  p.g = c.g;
  p.beta = c.beta;
  p.cu_seqlens = c.cu_seqlens;
  p.h0 = c.h0;
  p.hT = c.hT;
  p.o = c.o;
  p.seg = c.seg;
  p.h0_tab = c.h0_tab;
  p.hT_tab = c.hT_tab;
  p.v_zero = c.v_zero;
  p.h0_identity = c.h0_identity;
  p.flags = static_cast<uint32_t*>(c.workspace);
  p.ring = static_cast<uint8_t*>(c.workspace) + flag_bytes(S);
  p.gb_stride = c.gb_stride;
  p.num_seqs = c.num_seqs;
  p.total_tokens = c.total_tokens;
  p.H_k = c.H_k;
  p.H_v = c.H_v;
  p.D = D;
  p.S = S;
  p.scale = c.scale;
  p.spin_limit = g_spin_limit_override > 0 ? g_spin_limit_override : kSpinLimitCycles;
  // The hand-off counters start from zero on every launch.
  e = cudaMemsetAsync(c.workspace, 0, flag_bytes(S), s);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(G);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemAlloc;
  cfg.stream = s;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeCooperative;  // every CTA resident: spines and preps wait on each other
  attr.val.cooperative = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kernel, tq, tk, tv, to, p);
  if (e != cudaSuccess) return e;
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
