// Batched gathered FFN on the fifth-generation tensor cores (tcgen05).
//
// At a batch of B tokens the union of the tokens' predicted neurons
// (PowerInfer's neuron table, unite.ai page, "Neuronen-Platzierung und
// -Verwaltung") is a list of K neuron rows, and the neuron-aware operator
// (same page, "Neuronenbewusster Operator") becomes two small GEMMs over
// gathered rows:
//   up:   H[k][n]  = act(W_act[idx_k] . x_n (+ b), W_up[idx_k] . x_n)
//   down: y[n][c]  = sum_k H[k][n] W_down^T[idx_k][c]
// Both run here as tcgen05.mma (kind::f16, fp32 accumulation in tensor
// memory) on operands staged in 128-byte-swizzled shared memory:
//   - weight rows: four warps gather the listed rows, eight threads per
//     128-byte piece of a row.  16-bit pieces go straight into the swizzled
//     layout with 16-byte cp.async copies (no registers or L1 on the way);
//     Q4_0 blocks are loaded into registers, dequantized and stored.  Every
//     builder asks the L2 for its pieces a few stages ahead.  (A first
//     version gathered rows with cp.async.bulk.tensor .tile::gather4; at 128
//     bytes per row and four rows per instruction the copy engine delivered
//     about 1.7 TB/s, a quarter of what the copies here reach.)
//   - tokens (up) and H (down): 2-D tensor tiles copied by the tensor memory
//     accelerator, rows past the batch filled with zeros by the copy engine.
// One thread issues the copies, one thread the MMAs; the four builder warps
// then read the accumulator out of tensor memory (tcgen05.ld) for the
// epilogue.
//
// Precision: the products of 16-bit operands are exact and accumulate in
// fp32.  H is the one intermediate that must be rounded to a 16-bit MMA
// operand; it is split into hi = round16(h) and lo = round16(h - hi) and the
// down projection accumulates W.hi + W.lo, so H carries about 16 (bf16) or 22
// (fp16) significant bits -- enough to keep y within the 1e-3 budget.
//
// Shared-memory operand layouts (canonical tcgen05 SWIZZLE_128B forms):
//   K-major (rows of 64 16-bit values, 128 B; 8-row atoms of 1024 B; the
//   16-byte chunk c of row r stored at chunk c ^ (r % 8)): the up kernel's A
//   (neuron rows) and B (tokens), the down kernel's B (H rows per token).
//   MN-major (each W_down^T row segment of 64 columns is one 128-byte row of a
//   K-row atom): the down kernel's A, whose M index is the output column.
#pragma once
#include <cuda.h>

#include "pi_ffn.cuh"

namespace pi {

constexpr int kErrRange = 4;  // an fp16 H value overflowed (|h| > 65504)

// ---------------------------------------------------------------- tcgen05
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Warp-wide: allocate ncols (a power of two >= 32) tensor-memory columns; the
// address is written to *dst (shared memory).
__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst)),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
// D (tensor memory) (+)= A (smem descriptor) x B (smem descriptor).
__device__ __forceinline__ void umma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                         uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive once on *bar when every MMA this thread has issued so far completes.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}
// Warp-wide: 8 consecutive 32-bit columns of this warp's 32 tensor-memory
// lanes (thread i of the warp gets lane base + i).
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                 "=r"(r[6]), "=r"(r[7])
               : "r"(taddr)
               : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor, 128-byte swizzle (sm_100 format: start,
// leading and stride byte offsets in 16-byte units, version 1, layout 2).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}
// Instruction descriptor of kind::f16 with fp32 accumulation: operand type
// (0 fp16, 1 bf16), M x N, and whether A / B are MN-major.
template <int DT, int M, int N, int A_MN, int B_MN>
__host__ __device__ constexpr uint32_t idesc_f16() {
  return (1u << 4) | ((uint32_t)DT << 7) | ((uint32_t)DT << 10) | ((uint32_t)A_MN << 15) |
         ((uint32_t)B_MN << 16) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// ---------------------------------------------------------------- TMA
// One box of a 2-D tensor at (c0 = inner coordinate, c1 = row).
__device__ __forceinline__ void tma_load2d(void* dst, const CUtensorMap* tm, int c0, int c1,
                                           uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
      "l"(tm), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}

// ---------------------------------------------------------------- Q4_0
// The copy engine cannot dequantize, so with Q4_0 weights (DT 2) four warps
// build the weight operand themselves: each thread loads two consecutive
// blocks of a row (36 bytes, 4-byte aligned, as nine 32-bit words), turns
// them into 64 fp16 values (q - 8) * scale -- exact (q - 8) from the
// exponent trick 0x6400 | q = 1024 + q, then one rounding in the multiply by
// the block scale -- and stores them as eight 16-byte chunks in the swizzled
// layout.  The tensor cores then multiply fp16 x fp16 exactly with fp32
// accumulation; the one rounding of each weight (relative 2^-12 at most)
// keeps the FFN far inside its 2e-3 tolerance.
__device__ __forceinline__ void ld_q4_pair(const uint8_t* p, uint32_t (&w)[9]) {
  const uint32_t* q = reinterpret_cast<const uint32_t*>(p);
#pragma unroll
  for (int k = 0; k < 9; ++k) w[k] = __ldg(q + k);
}

// Two fp16 values (q - 8) * scale for the nibbles q held in two bytes of v
// (each byte 0..15; sel picks them: 0x4140 bytes 0-1, 0x4342 bytes 2-3).
// The pair stays packed in one 32-bit register: a byte permute makes the
// halves 0x6400 | q = 1024 + q, a packed subtract of 1032 leaves q - 8
// exactly, and a packed multiply by the scale pair rounds once.  (Unpacking
// to two halves and repacking cost about three times the instructions, and
// the operand builders were issue-bound on it.)
__device__ __forceinline__ uint32_t q4_h2(uint32_t v, uint32_t sel, uint32_t scale2) {
  const uint32_t biased = __byte_perm(v, 0x64646464u, sel);
  uint32_t r;
  asm("{\n\t.reg .b32 t;\n\t"
      "sub.rn.f16x2 t, %1, %3;\n\t"
      "mul.rn.f16x2 %0, t, %2;\n\t}"
      : "=r"(r)
      : "r"(biased), "r"(scale2), "r"(0x64086408u));
  return r;
}

// 36 bytes = blocks A and B -> chunks c = 0..7 of 8 consecutive values each
// (chunks 0-3 from block A, 4-7 from block B; within a block chunk 0 is the
// low nibbles of bytes 0-7, chunk 1 of bytes 8-15, chunks 2-3 the high ones).
__device__ __forceinline__ void dq_q4_pair(const uint32_t (&w)[9], uint4 (&out)[8]) {
#pragma unroll
  for (int b = 0; b < 2; ++b) {
    uint32_t nb[4];
    uint32_t sbits;
    if (b == 0) {
      sbits = w[0] & 0xffffu;
#pragma unroll
      for (int k = 0; k < 4; ++k) nb[k] = __funnelshift_r(w[k], w[k + 1], 16);
    } else {
      sbits = w[4] >> 16;
#pragma unroll
      for (int k = 0; k < 4; ++k) nb[k] = w[5 + k];
    }
    const uint32_t s2 = sbits | (sbits << 16);  // the block scale in both halves
    uint32_t lo[4], hi[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      lo[k] = nb[k] & 0x0F0F0F0Fu;
      hi[k] = (nb[k] >> 4) & 0x0F0F0F0Fu;
    }
    out[4 * b + 0] = make_uint4(q4_h2(lo[0], 0x4140u, s2), q4_h2(lo[0], 0x4342u, s2),
                                q4_h2(lo[1], 0x4140u, s2), q4_h2(lo[1], 0x4342u, s2));
    out[4 * b + 1] = make_uint4(q4_h2(lo[2], 0x4140u, s2), q4_h2(lo[2], 0x4342u, s2),
                                q4_h2(lo[3], 0x4140u, s2), q4_h2(lo[3], 0x4342u, s2));
    out[4 * b + 2] = make_uint4(q4_h2(hi[0], 0x4140u, s2), q4_h2(hi[0], 0x4342u, s2),
                                q4_h2(hi[1], 0x4140u, s2), q4_h2(hi[1], 0x4342u, s2));
    out[4 * b + 3] = make_uint4(q4_h2(hi[2], 0x4140u, s2), q4_h2(hi[2], 0x4342u, s2),
                                q4_h2(hi[3], 0x4140u, s2), q4_h2(hi[3], 0x4342u, s2));
  }
}

// ---------------------------------------------------------------- kernels
constexpr int kUmmaThreads = 192;  // warp 0 copies, warp 1 MMAs, warps 2-5 epilogue
constexpr int kUmmaDownThreads = 224;  // the down kernel adds warp 6, its L2 prefetcher
// Stages of raw Q4_0 blocks the down kernel's builders keep in flight in
// registers (36 bytes per thread per stage).
constexpr int kQ4DownAhead = 4;
constexpr int kUmmaM = 128;        // neuron rows (up) / output columns (down) per tile
constexpr int kUmmaK = 64;         // contraction elements per stage (one 128-byte row)

struct UmmaParams {
  const int32_t* idx;      // neuron list (first *count entries) ...
  const int32_t* count;
  const uint32_t* mask;    // ... or, up kernel: the predictor's mask rows
  int mask_rows;           //   [mask_rows x F/32], whose OR is the list; the
  int32_t* idx_out;        //   tiles' ids are written to idx_out and the
  int32_t* count_out;      //   length to count_out
  const uint8_t* wa;       // Q4_0 rows (DT 2): activation rows (W_up or W_gate) ...
  const uint8_t* wa2;      // ... W_up rows (ReGLU) ...
  const uint8_t* wd;       // ... and W_down^T rows
  uint32_t rb;             // bytes of one Q4_0 row
  const float* bias;       // up: b_up (ReLU, Squared-ReLU) or b_gate (ReGLU), or null
  uint16_t* hh;            // [B x F] 16-bit hi part of H (token-major)
  uint16_t* hl;            // [B x F] 16-bit lo part
  float* part;             // down: [gridDim.y x B x d] partial y
  float* pu;               // up, contraction split in S slices: per (tile, slice)
                           //   unit, [NMAT x B x 128] fp32 accumulators
  int ucap;                // up: most units (grid size, room in pu)
  int slots;               // up: CTAs resident at once (two per SM)
  int d, F, B;
};

// Slices of the contraction per 128-row tile of the up projection.  With T
// tiles listed, S slices give T * S units of 1/S of a tile's work each; the
// pick minimises ceil(T S / slots) / S (waves times the work of a unit) over
// S = 1..8 (ties to fewer slices), with T S <= ucap and at least 8 stages in
// a slice.  Slices are whole granules of gran stages.  The up kernel and its
// finishing kernel both call this, so they agree on S.
__host__ __device__ inline int up_slices(int T, int ucap, int slots, int ngran, int gran) {
  int best = 1;
  long long bw = (T + slots - 1) / slots;  // waves with one slice
  for (int S = 2; S <= 8; ++S) {
    if ((long long)T * S > ucap || (ngran / S) * gran < 8) break;
    const long long w = ((long long)T * S + slots - 1) / slots;
    if (w * best < bw * S) {
      best = S;
      bw = w;
    }
  }
  return best;
}

// Bytes of one pipeline stage.
template <int NMAT, int N>
__host__ __device__ constexpr int umma_up_stage() {
  return NMAT * kUmmaM * kUmmaK * 2 + N * kUmmaK * 2;
}
template <int N>
__host__ __device__ constexpr int umma_down_stage() {
  return kUmmaM * kUmmaK * 2 + 2 * N * kUmmaK * 2;
}

// Round an fp32 value to the 16-bit MMA type (nearest even) and back.
template <int DT>
__device__ __forceinline__ uint16_t to16(float v) { return round16<DT>(v); }
template <int DT>
__device__ __forceinline__ float from16(uint16_t u) {
  if constexpr (DT == 0) return __half2float(__ushort_as_half(u));
  else return __uint_as_float((uint32_t)u << 16);
}

// L2 prefetch of the line holding p: the operand builders ask for the
// weight pieces of stage i + kPfAhead while they work on stage i, so the
// copies and loads of a stage find their lines in the L2.  Measured on the
// batched kernels: dropping it costs 10-30%; for the 16-bit builders, whose
// asynchronous copies are already up to six stages ahead, 4 stages beat 8
// by 3-7% (12 and 16 are slower); the Q4_0 builders, which load a
// super-stage at a time into registers, want 8 (two super-stages).
// Bursts of a row's pieces and evict-last priority gain nothing.
constexpr int kPfAhead = 4;
constexpr int kPfAheadQ4 = 8;
__device__ __forceinline__ void prefetch_line(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// 16-byte asynchronous copy global -> shared that bypasses the L1 (so the
// bytes in flight are bounded by the pipeline's stage buffers, not by the L1
// left over after the shared-memory carve-out), with an L2 policy (the
// builders pass evict-first: each row piece is read once, and without the
// hint the consumed lines crowded out prefetched ones, 1.46x the bytes from
// DRAM on the 13B up projection), and the arrive on an mbarrier once all of
// this thread's earlier copies have landed (.noinc: the barrier's expected
// count includes these arrivals).  The consumer fences the async proxy
// after its wait, before the tensor cores read the stage.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint64_t pol) {
  asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "l"(pol)
               : "memory");
}
// Same, reading src_bytes (0 or 16) and filling the rest of the 16 with zeros.
__device__ __forceinline__ void cp_async16_fill(uint32_t dst, const void* src, uint32_t src_bytes,
                                                uint64_t pol) {
  asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2, %3;" ::"r"(dst),
               "l"(src), "r"(src_bytes), "l"(pol)
               : "memory");
}
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_all;" ::: "memory");
}


// One activation of the up projection: h = act(a + bias) (ReGLU: times the
// up row's sum u), written as the hi and lo 16-bit parts of H (type HT) at
// token n, list position k; zero where the position holds no neuron.
template <int HT, int ACT>
__device__ __forceinline__ void up_store(const UmmaParams& p, int n, int k, float a, float u,
                                         float bias, bool live) {
  float h = 0.f;
  if (live) {
    const float r = fmaxf(a + bias, 0.f);
    h = ACT == 1 ? r * u : ACT == 2 ? r * r : r;
  }
  const uint16_t hi = to16<HT>(h);
  const float fh = from16<HT>(hi);
  if (HT == 0 && isinf(fh)) set_error(kErrRange);
  p.hh[(size_t)n * p.F + k] = hi;
  p.hl[(size_t)n * p.F + k] = to16<HT>(h - fh);
}

// Gathered up projection + activation.  The work is T tiles of 128 listed
// neurons (T from the device-side count), each split into S slices of the
// contraction over d (up_slices: S > 1 when T alone would leave SMs idle);
// CTA u takes tile u / S, slice u % S, and CTAs past T S exit at once.  A
// slice runs in stages of 64 elements.  With S = 1 the CTA applies the
// activation itself; with S > 1 it writes its raw sums to pu and
// k_umma_up_finish completes the tile.  DT: 0 fp16, 1 bf16 (weights and tokens),
// 2 Q4_0 weights with fp16 tokens.  ACT: 0 ReLU, 1 ReGLU (gate rows in p.wa,
// up rows in p.wa2), 2 Squared-ReLU.  N: tokens per MMA (the batch rounded up
// to a multiple of 16).
//   warp 0     copies the stage's token tile (TMA, rows past the batch zero)
//   warp 1     issues the MMAs (one thread) and owns the tensor memory
//   warps 2-5  build the weight operand: the tile's 128 gathered rows, 64
//              elements per stage, 8 threads per 128-byte row piece (16-bit
//              rows: asynchronous copies straight into the swizzled layout;
//              Q4_0: loads, decode, stores); then the epilogue
template <int DT, int ACT, int N, int NS>
__global__ void __launch_bounds__(kUmmaThreads, 2)
    k_umma_up(const __grid_constant__ CUtensorMap tm_x, UmmaParams p) {
  constexpr int NMAT = ACT == 1 ? 2 : 1;
  constexpr bool Q4 = DT == 2;
  constexpr int ABYTES = kUmmaM * kUmmaK * 2;  // 16 KB per matrix
  constexpr int STAGE = umma_up_stage<NMAT, N>();
  constexpr uint32_t NCOL = NMAT * N <= 32 ? 32 : NMAT * N <= 64 ? 64 : NMAT * N <= 128 ? 128 : 256;
  constexpr uint32_t IDESC = idesc_f16<Q4 ? 0 : DT, kUmmaM, N, 0, 0>();
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  __shared__ uint64_t full[NS], empty[NS], done;
  __shared__ uint32_t tmem_base;
  __shared__ int ids[kUmmaM];
  __shared__ float bias_s[kUmmaM];

  pdl_wait();
  pdl_trigger();
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  int K;
  // mask mode: the list is the ascending union of the mask rows; every CTA
  // scans it (in the stage buffers, not yet in use)
  const uint32_t* wmask = reinterpret_cast<const uint32_t*>(smem);
  const int* wpre = reinterpret_cast<const int*>(smem) + p.F / 32;
  if (p.mask) {
    __shared__ int scan_tmp[33];
    const int W = p.F / 32;
    uint32_t* wm = reinterpret_cast<uint32_t*>(smem);
    int* wp = reinterpret_cast<int*>(smem) + W;
    const int wpt = (W + kUmmaThreads - 1) / kUmmaThreads;
    int mine = 0;
    for (int k = 0; k < wpt; ++k) {
      const int w = t * wpt + k;
      if (w < W) {
        uint32_t m = 0u;
        for (int b = 0; b < p.mask_rows; ++b) m |= p.mask[(size_t)b * W + w];
        wm[w] = m;
        mine += __popc(m);
      }
    }
    int pos = block_excl_scan<kUmmaThreads>(mine, scan_tmp, K);
    for (int k = 0; k < wpt; ++k) {
      const int w = t * wpt + k;
      if (w < W) {
        wp[w] = pos;
        pos += __popc(wm[w]);
      }
    }
    __syncthreads();
    if (blockIdx.x == 0 && t == 0) *p.count_out = K;
  } else {
    K = *p.count;
    K = K < 0 ? 0 : (K > p.F ? p.F : K);
  }
  // this CTA's unit: tile of 128 listed neurons, slice of the contraction
  constexpr int GRAN = Q4 ? 4 : 1;  // Q4_0 rows are read 4 stages (144 B) at a time
  const int ngran = p.d / kUmmaK / GRAN;
  const int T = (K + kUmmaM - 1) / kUmmaM;
  const int S = up_slices(T, p.ucap, p.slots, ngran, GRAN);
  const int tile = blockIdx.x / S, slice = blockIdx.x - tile * S;
  if (tile >= T) return;  // whole CTA
  const int k0 = tile * kUmmaM;
  const int st0 = ngran * slice / S * GRAN;
  const int nst = ngran * (slice + 1) / S * GRAN - st0;
  if (t < kUmmaM) {
    int id = -1;
    if (k0 + t < K) {
      const int q = k0 + t;
      if (p.mask) {
        int lo = 0, hi = p.F / 32 - 1;  // the last word whose prefix is <= q
        while (lo < hi) {
          const int mid = (lo + hi + 1) >> 1;
          if (wpre[mid] <= q) lo = mid;
          else hi = mid - 1;
        }
        id = lo * 32 + (int)__fns(wmask[lo], 0, q - wpre[lo] + 1);
        if (slice == 0) p.idx_out[q] = id;
      } else {
        id = p.idx[q];
        if (id < 0 || id >= p.F) {
          set_error(kErrBadIndex);
          id = -1;
        }
      }
    }
    ids[t] = id;
    bias_s[t] = (id >= 0 && p.bias) ? p.bias[id] : 0.f;
  }
  __syncthreads();  // the scan scratch is reused as stage buffers below
  if (t == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1 + kUmmaM);  // the token copy + 128 builder threads
      mbar_init(&empty[s], 1);
    }
    mbar_init(&done, 1);
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(&tmem_base, NCOL);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;

  if (warp == 0) {
    if (lane == 0) {  // token tiles
      for (int i = 0; i < nst; ++i) {
        const int s = i % NS;
        if (i >= NS && !mbar_wait(&empty[s], ((i / NS) - 1) & 1)) break;
        mbar_arrive_expect_tx(&full[s], N * kUmmaK * 2);
        tma_load2d(smem + (size_t)s * STAGE + NMAT * ABYTES, &tm_x, (st0 + i) * kUmmaK, 0,
                   &full[s]);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {  // MMA issuer
      for (int i = 0; i < nst; ++i) {
        const int s = i % NS;
        if (!mbar_wait(&full[s], (i / NS) & 1)) break;
        if constexpr (!Q4) fence_proxy_async_smem();  // the builders' async copies
        tc_fence_after();
        const uint32_t sa = smem_u32(smem + (size_t)s * STAGE);
        const uint32_t sb = sa + NMAT * ABYTES;
#pragma unroll
        for (int kk = 0; kk < kUmmaK / 16; ++kk) {  // 16 elements = 32 bytes per MMA
          const uint64_t bd = sw128_desc(sb + 32 * kk, 16, 1024);
          umma_f16(tmem, sw128_desc(sa + 32 * kk, 16, 1024), bd, IDESC, (i | kk) != 0);
          if constexpr (NMAT == 2)
            umma_f16(tmem + N, sw128_desc(sa + ABYTES + 32 * kk, 16, 1024), bd, IDESC,
                     (i | kk) != 0);
        }
        umma_commit(&empty[s]);
      }
      umma_commit(&done);
    }
    __syncwarp();
  } else {
    const int m = t - 64;  // 0..127
    bool ok = true;
    if constexpr (Q4) {
      // thread m builds row m.  It loads a super-stage at a time: eight
      // blocks = 144 bytes = four MMA stages of its row, with nine 128-bit
      // loads (row pieces of 144 bytes stay 16-byte aligned since d % 256 ==
      // 0), and decodes two blocks per stage from registers.  (Loading two
      // blocks per stage as nine 32-bit words made every warp instruction
      // touch 32 rows for 4 bytes each, and the L1 request rate, not HBM,
      // set the pace.)  The L2 is asked for the pieces two super-stages ahead.
      const int id = max(ids[m], 0);
      const size_t roff = (size_t)id * p.rb + (size_t)(st0 / 4) * 144;  // the slice's first block
      const uint8_t* rowp[NMAT];
      rowp[0] = p.wa + roff;
      if constexpr (NMAT == 2) rowp[NMAT - 1] = p.wa2 + roff;
      const int nss = nst / 4;  // super-stages
      constexpr int SSA = kPfAheadQ4 / 4;
      auto pf_ss = [&](int ss) {
#pragma unroll
        for (int mm = 0; mm < NMAT; ++mm) {
          prefetch_line(rowp[mm] + 144 * ss);
          prefetch_line(rowp[mm] + 144 * ss + 143);
        }
      };
      for (int ss = 1; ss <= SSA && ss < nss; ++ss) pf_ss(ss);
      const uint32_t rsw = (uint32_t)(m & 7);
      uint32_t raw[NMAT][36];
      auto ld_ss = [&](int ss) {
#pragma unroll
        for (int mm = 0; mm < NMAT; ++mm) {
          const uint4* src = reinterpret_cast<const uint4*>(rowp[mm] + 144 * ss);
#pragma unroll
          for (int k = 0; k < 9; ++k) {
            const uint4 v = __ldg(src + k);
            raw[mm][4 * k] = v.x; raw[mm][4 * k + 1] = v.y;
            raw[mm][4 * k + 2] = v.z; raw[mm][4 * k + 3] = v.w;
          }
        }
      };
      if (nss > 0) ld_ss(0);
      for (int ss = 0; ss < nss && ok; ++ss) {
        if (ss + SSA + 1 < nss) pf_ss(ss + SSA + 1);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int i = 4 * ss + u;
          const int s = i % NS;
          if (ok && i >= NS && !mbar_wait(&empty[s], ((i / NS) - 1) & 1)) ok = false;
          if (ok) {
            uint8_t* row0 = smem + (size_t)s * STAGE + (m >> 3) * 1024 + (m & 7) * 128;
#pragma unroll
            for (int mm = 0; mm < NMAT; ++mm) {
              uint32_t w[9];
#pragma unroll
              for (int k = 0; k < 9; ++k) w[k] = raw[mm][9 * u + k];
              uint4 ch[8];
              dq_q4_pair(w, ch);
#pragma unroll
              for (int c = 0; c < 8; ++c)
                *reinterpret_cast<uint4*>(row0 + mm * ABYTES + ((c ^ rsw) << 4)) = ch[c];
            }
            fence_proxy_async_smem();
            mbar_arrive(&full[s]);
          }
        }
        if (ss + 1 < nss && ok) ld_ss(ss + 1);
      }
    } else {
      // 16-bit rows: thread m takes chunk c = m % 8 (16 bytes) of rows
      // 8 (m / 8) + j, j = 0..7, i.e. row j of 8-row group m / 8, and copies
      // its eight pieces of each stage straight into the swizzled layout
      // (cp.async, no registers or L1 on the way): up to NS stages in flight
      const int c = m & 7, g = m >> 3;
      const uint8_t* rowp[NMAT][8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const size_t off = (size_t)max(ids[8 * g + j], 0) * p.rb + (size_t)st0 * 128 + (size_t)c * 16;
        rowp[0][j] = p.wa + off;
        if constexpr (NMAT == 2) rowp[NMAT - 1][j] = p.wa2 + off;
      }
      // prefetch: thread m asks for row m's 128-byte piece of each stage
      const uint8_t* pfrow[NMAT];
      {
        const size_t off = (size_t)max(ids[m], 0) * p.rb + (size_t)st0 * 128;
        pfrow[0] = p.wa + off;
        if constexpr (NMAT == 2) pfrow[NMAT - 1] = p.wa2 + off;
      }
      for (int j = 0; j < kPfAhead && j < nst; ++j)
#pragma unroll
        for (int mm = 0; mm < NMAT; ++mm) prefetch_line(pfrow[mm] + 128 * j);
      const uint32_t gb = smem_u32(smem + g * 1024);
      const uint64_t pol = policy_evict_first();  // a row piece is read once
      for (int i = 0; i < nst; ++i) {
        const int s = i % NS;
        if (i + kPfAhead < nst)
#pragma unroll
          for (int mm = 0; mm < NMAT; ++mm) prefetch_line(pfrow[mm] + 128 * (i + kPfAhead));
        if (i >= NS && !mbar_wait(&empty[s], ((i / NS) - 1) & 1)) {
          ok = false;
          break;
        }
        const uint32_t st = gb + (uint32_t)(s * STAGE);
#pragma unroll
        for (int mm = 0; mm < NMAT; ++mm)
#pragma unroll
          for (int j = 0; j < 8; ++j)
            cp_async16(st + (uint32_t)(mm * ABYTES + j * 128 + ((c ^ j) << 4)),
                       rowp[mm][j] + 128 * i, pol);
        cp_async_arrive_noinc(&full[s]);
      }
      cp_async_wait_all();
    }
    // epilogue: warp w reads tensor-memory lanes 32 (w % 4) .. + 31 (neurons)
    const int quad = warp & 3;
    const int mr = quad * 32 + lane;
    const bool done_ok = mbar_wait_sleep(&done, 0);
    tc_fence_after();
    const int k = k0 + mr;
    const int id = ids[mr];
    const float bias = bias_s[mr];
    // with S > 1 slices the unit's raw sums go to pu[unit] ([NMAT x B x 128]);
    // k_umma_up_finish adds the slices and applies the activation
    float* pu = p.pu + (size_t)blockIdx.x * NMAT * p.B * kUmmaM;
#pragma unroll
    for (int c0 = 0; c0 < N; c0 += 8) {
      uint32_t ra[8], ru[8];
      tmem_ld8(tmem + ((uint32_t)(quad * 32) << 16) + c0, ra);
      if constexpr (NMAT == 2) tmem_ld8(tmem + ((uint32_t)(quad * 32) << 16) + N + c0, ru);
      tmem_wait_ld();
      if (S > 1) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int n = c0 + j;
          if (n < p.B) {
            const bool live = ok && done_ok;
            pu[(size_t)n * kUmmaM + mr] = live ? __uint_as_float(ra[j]) : 0.f;
            if constexpr (NMAT == 2)
              pu[(size_t)(p.B + n) * kUmmaM + mr] = live ? __uint_as_float(ru[j]) : 0.f;
          }
        }
      } else if (k < p.F) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int n = c0 + j;
          if (n < p.B)
            up_store<Q4 ? 0 : DT, ACT>(p, n, k, __uint_as_float(ra[j]),
                                       NMAT == 2 ? __uint_as_float(ru[j]) : 0.f, bias,
                                       ok && done_ok && id >= 0);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, NCOL);
  }
}

// Completes a split up projection: for every listed position k of the T
// tiles and token n, adds the S slices' sums in slice order, applies bias
// and activation and writes H (up_store).  Recomputes S as the up kernel
// did, and exits at once when S = 1.  Grid-stride over T x B x 128.
template <int DT, int ACT>
__global__ void __launch_bounds__(256) k_umma_up_finish(UmmaParams p) {
  constexpr int NMAT = ACT == 1 ? 2 : 1;
  constexpr int GRAN = DT == 2 ? 4 : 1;
  pdl_wait();
  pdl_trigger();
  int K = *(p.mask ? p.count_out : p.count);
  K = K < 0 ? 0 : (K > p.F ? p.F : K);
  const int T = (K + kUmmaM - 1) / kUmmaM;
  const int S = up_slices(T, p.ucap, p.slots, p.d / kUmmaK / GRAN, GRAN);
  if (S == 1) return;
  const int32_t* list = p.mask ? p.idx_out : p.idx;
  const size_t total = (size_t)T * p.B * kUmmaM;
  for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < total;
       e += (size_t)gridDim.x * blockDim.x) {
    const int m = (int)(e % kUmmaM);
    const int n = (int)((e / kUmmaM) % p.B);
    const int tile = (int)(e / ((size_t)kUmmaM * p.B));
    const int k = tile * kUmmaM + m;
    if (k >= p.F) continue;
    int id = k < K ? list[k] : -1;
    if (id < 0 || id >= p.F) id = -1;  // a bad id was flagged by the up kernel
    float a = 0.f, u = 0.f;
    if (id >= 0) {
      for (int sl = 0; sl < S; ++sl) {
        const float* src = p.pu + (size_t)(tile * S + sl) * NMAT * p.B * kUmmaM;
        a += src[(size_t)n * kUmmaM + m];
        if constexpr (NMAT == 2) u += src[(size_t)(p.B + n) * kUmmaM + m];
      }
    }
    const float bias = (id >= 0 && p.bias) ? p.bias[id] : 0.f;
    up_store<DT == 2 ? 0 : DT, ACT>(p, n, k, a, u, bias, id >= 0);
  }
}

// Gathered down projection.  Grid (d / 128 column tiles, S neuron slices);
// CTA (c, s) sums the neuron positions of slice s (stages of 64) into the
// 128 x N accumulator of columns [128c, 128c + 128) and writes it to
// part[s].  Positions past the list hold H = 0 (the up kernel writes zeros
// up to the next multiple of 128), and their weight rows are taken from row 0.
//   warp 0     copies the stage's H tiles, hi and lo (TMA)
//   warp 1     issues the MMAs and owns the tensor memory
//   warps 2-5  build the weight operand: 64 neurons x 128 columns per stage,
//              each neuron's 256-byte row segment taken by 16 threads (16-bit:
//              asynchronous copies), stored as one 128-byte row in each of
//              the two column atoms (MN-major, swizzled); then the epilogue.
//              Q4_0: loads and decode in registers, two threads per neuron
//   warp 6     reads the neuron ids of the stages ahead and asks the L2 for
//              their row segments, at most kPfAhead (Q4_0: kPfAheadQ4) stages ahead of the MMAs
//              (which publish their progress in shared memory); the ids it
//              reads are then in the L1 for the builders
template <int DT, int N, int NS>
__global__ void __launch_bounds__(kUmmaDownThreads, 2)
    k_umma_down(const __grid_constant__ CUtensorMap tm_hh, const __grid_constant__ CUtensorMap tm_hl,
                UmmaParams p) {
  constexpr bool Q4 = DT == 2;
  constexpr int ABYTES = kUmmaM * kUmmaK * 2;  // 2 column atoms of 64 neurons x 128 B
  constexpr int BBYTES = N * kUmmaK * 2;
  constexpr int STAGE = umma_down_stage<N>();
  constexpr uint32_t NCOL = N <= 32 ? 32 : N <= 64 ? 64 : N <= 128 ? 128 : 256;
  constexpr uint32_t IDESC = idesc_f16<Q4 ? 0 : DT, kUmmaM, N, 1, 0>();
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  __shared__ uint64_t full[NS], empty[NS], done;
  __shared__ uint32_t tmem_base;
  __shared__ int prog;  // the last stage whose operands the MMA thread has seen

  pdl_wait();
  pdl_trigger();
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  if (t == 0) prog = -1;
  int K = *p.count;
  K = K < 0 ? 0 : (K > p.F ? p.F : K);
  const int T = (K + kUmmaK - 1) / kUmmaK;  // stages of the whole list
  const int S = gridDim.y;
  const int st0 = (int)(((long long)T * blockIdx.y) / S);
  const int st1 = (int)(((long long)T * (blockIdx.y + 1)) / S);
  const int nst = st1 - st0;
  const int col0 = blockIdx.x * kUmmaM;
  if (t == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1 + kUmmaM);  // the H copies + 128 builder threads
      mbar_init(&empty[s], 1);
    }
    mbar_init(&done, 1);
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(&tmem_base, NCOL);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;

  if (warp == 0) {
    if (lane == 0) {  // H tiles
      for (int i = 0; i < nst; ++i) {
        const int s = i % NS;
        if (i >= NS && !mbar_wait(&empty[s], ((i / NS) - 1) & 1)) break;
        uint8_t* st = smem + (size_t)s * STAGE;
        mbar_arrive_expect_tx(&full[s], 2 * BBYTES);
        tma_load2d(st + ABYTES, &tm_hh, (st0 + i) * kUmmaK, 0, &full[s]);
        tma_load2d(st + ABYTES + BBYTES, &tm_hl, (st0 + i) * kUmmaK, 0, &full[s]);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {  // MMA issuer
      for (int i = 0; i < nst; ++i) {
        const int s = i % NS;
        if (!mbar_wait(&full[s], (i / NS) & 1)) break;
        *reinterpret_cast<volatile int*>(&prog) = i;
        if constexpr (!Q4) fence_proxy_async_smem();  // the builders' async copies
        tc_fence_after();
        const uint32_t sa = smem_u32(smem + (size_t)s * STAGE);
        const uint32_t sh = sa + ABYTES, sl = sh + BBYTES;
#pragma unroll
        for (int kk = 0; kk < kUmmaK / 16; ++kk) {
          // A: 16 neurons = two 8-row groups of 1024 B; the second 64 columns
          // sit ABYTES / 2 further on
          const uint64_t ad = sw128_desc(sa + 2048 * kk, ABYTES / 2, 1024);
          umma_f16(tmem, ad, sw128_desc(sh + 32 * kk, 16, 1024), IDESC, (i | kk) != 0);
          umma_f16(tmem, ad, sw128_desc(sl + 32 * kk, 16, 1024), IDESC, 1);
        }
        umma_commit(&empty[s]);
      }
      umma_commit(&done);
    }
    __syncwarp();
  } else if (warp == 6) {
    // the L2 prefetcher: lane l takes neurons 2l and 2l + 1 of each stage
    const size_t coff = Q4 ? (size_t)(col0 / 32) * 18 : (size_t)col0 * 2;
    const int span = Q4 ? 71 : 255;  // last byte of a neuron's segment
    for (int j = 0; j < nst; ++j) {
      uint32_t it = 0;
      while (*reinterpret_cast<volatile int*>(&prog) < j - (Q4 ? kPfAheadQ4 : kPfAhead) &&
             ++it < kWaitLimitSleep)
        __nanosleep(128);
      if (it >= kWaitLimitSleep) break;  // only a hint: stop prefetching
      const int kp = (st0 + j) * kUmmaK + 2 * lane;
      int ia = -1, ib = -1;
      if (kp + 1 < K) {
        const int2 v = __ldg(reinterpret_cast<const int2*>(p.idx + kp));
        ia = v.x;
        ib = v.y;
      } else if (kp < K) {
        ia = p.idx[kp];
      }
      if (ia >= 0 && ia < p.F) {
        const uint8_t* r = p.wd + (size_t)ia * p.rb + coff;
        prefetch_line(r);
        prefetch_line(r + span);
      }
      if (ib >= 0 && ib < p.F) {
        const uint8_t* r = p.wd + (size_t)ib * p.rb + coff;
        prefetch_line(r);
        prefetch_line(r + span);
      }
    }
  } else {
    const int m = t - 64;  // 0..127
    bool ok = true;
    if constexpr (Q4) {
      // thread m takes neuron m / 2 of each stage and columns
      // [64 (m % 2), 64 (m % 2) + 64) of the tile: two blocks, which become one
      // 128-byte row of column atom m % 2
      const int kk = m >> 1, half = m & 1;
      const size_t coff = (size_t)(col0 / 32) * 18 + 36 * half;
      auto row_of = [&](int i) -> const uint8_t* {
        const int kp = (st0 + i) * kUmmaK + kk;
        int id = kp < K ? p.idx[kp] : -1;
        if (id < 0 || id >= p.F) id = -1;  // flagged by the up kernel; zero row
        return id < 0 ? nullptr : p.wd + (size_t)id * p.rb + coff;
      };
      constexpr int QA = kQ4DownAhead;
      uint32_t raw[QA][9];
      bool live[QA];
#pragma unroll
      for (int j = 0; j < QA; ++j) {
        const uint8_t* r = j < nst ? row_of(j) : nullptr;
        live[j] = r != nullptr;
        if (r) ld_q4_pair(r, raw[j]);
      }
      const uint32_t rsw = (uint32_t)(kk & 7);
      for (int i0 = 0; i0 < nst && ok; i0 += QA) {
#pragma unroll
        for (int j = 0; j < QA; ++j) {
          const int i = i0 + j;
          if (i < nst && ok) {
            const int s = i % NS;
            if (i >= NS && !mbar_wait(&empty[s], ((i / NS) - 1) & 1)) ok = false;
            if (ok) {
              uint8_t* row0 = smem + (size_t)s * STAGE + half * (ABYTES / 2) + (kk >> 3) * 1024 +
                              (kk & 7) * 128;
              uint4 ch[8];
              if (live[j]) {
                dq_q4_pair(raw[j], ch);
              } else {
#pragma unroll
                for (int c = 0; c < 8; ++c) ch[c] = make_uint4(0, 0, 0, 0);
              }
#pragma unroll
              for (int c = 0; c < 8; ++c) *reinterpret_cast<uint4*>(row0 + ((c ^ rsw) << 4)) = ch[c];
              fence_proxy_async_smem();
              mbar_arrive(&full[s]);
              if (i + QA < nst) {
                const uint8_t* r = row_of(i + QA);
                live[j] = r != nullptr;
                if (r) ld_q4_pair(r, raw[j]);
              }
            }
          }
        }
      }
    } else {
      // 16-bit rows: thread m takes column chunk c = m % 16 (8 columns) of
      // neurons 8 (m / 16) + j, j = 0..7 of the stage, copied straight into
      // the swizzled layout (cp.async); the next stage's ids are read while
      // this stage's copies are in flight
      const int c = m & 15, g = m >> 4;
      const uint8_t* cbase = p.wd + (size_t)(col0 + 8 * c) * 2;
      auto ids_of = [&](int i, int (&id)[8]) {
        const int kp = (st0 + i) * kUmmaK + 8 * g;
        if (kp + 8 <= K) {
          const int4 a = __ldg(reinterpret_cast<const int4*>(p.idx + kp));
          const int4 b = __ldg(reinterpret_cast<const int4*>(p.idx + kp + 4));
          id[0] = a.x; id[1] = a.y; id[2] = a.z; id[3] = a.w;
          id[4] = b.x; id[5] = b.y; id[6] = b.z; id[7] = b.w;
        } else {
#pragma unroll
          for (int j = 0; j < 8; ++j) id[j] = kp + j < K ? p.idx[kp + j] : 0;
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) id[j] = (id[j] < 0 || id[j] >= p.F) ? 0 : id[j];
      };
      int idn[8];
      if (nst > 0) ids_of(0, idn);
      const int cc = c & 7;
      const uint32_t gb = smem_u32(smem + (c >> 3) * (ABYTES / 2) + g * 1024);
      const uint64_t pol = policy_evict_first();
      for (int i = 0; i < nst; ++i) {
        const int s = i % NS;
        if (i >= NS && !mbar_wait(&empty[s], ((i / NS) - 1) & 1)) {
          ok = false;
          break;
        }
        const uint32_t st = gb + (uint32_t)(s * STAGE);
#pragma unroll
        for (int j = 0; j < 8; ++j)
          cp_async16(st + (uint32_t)(j * 128 + ((cc ^ j) << 4)), cbase + (size_t)idn[j] * p.rb, pol);
        cp_async_arrive_noinc(&full[s]);
        if (i + 1 < nst) ids_of(i + 1, idn);
      }
      cp_async_wait_all();
    }
    const int quad = warp & 3;
    const int col = col0 + quad * 32 + lane;  // output column of this lane
    const bool done_ok = nst == 0 || mbar_wait_sleep(&done, 0);
    tc_fence_after();
#pragma unroll
    for (int c0 = 0; c0 < N; c0 += 8) {
      uint32_t r[8];
      if (nst > 0) {
        tmem_ld8(tmem + ((uint32_t)(quad * 32) << 16) + c0, r);
        tmem_wait_ld();
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int n = c0 + j;
        if (n < p.B && col < p.d)
          p.part[((size_t)blockIdx.y * p.B + n) * p.d + col] =
              (nst > 0 && ok && done_ok) ? __uint_as_float(r[j]) : 0.f;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, NCOL);
  }
}

// The predictor on the tensor cores, at batches of 16 or more (a dense
// contraction there).  Both layers read every row of their matrix (no
// gather): one CTA per 128 rows, the contraction in stages of 64.
//   layer 2 (L1 = false): s = W2 a + b2 and the threshold.  The hidden
//     activations a (fp32) enter as the hi + lo pair of 16-bit values written
//     by layer 1.  In the epilogue a warp holds 32 consecutive neurons, one
//     per lane, so a ballot over the warp is exactly one mask word per token:
//     the mask is written whole, with no atomics, and so is the OR of the
//     batch's words (the union the FFN compacts).
//   layer 1 (L1 = true): W1 x, split over the contraction (gridDim.y slices,
//     the rank has only rank/128 tiles); each CTA writes its fp32 partial and
//     k_pred1_finish sums the slices in order and applies b1 and the ReLU.
//   warp 0     copies the stage's activation tiles (TMA): a hi and lo, or x
//   warp 1     issues the MMAs and owns the tensor memory
//   warps 2-5  copy the stage's weight rows (8 threads per 128-byte row
//              piece, cp.async) into the swizzled layout; then the epilogue
struct UmmaPredParams {
  const uint8_t* w;        // [nrows x len] 16-bit rows (W2 or W1)
  const float* bias;       // b2 (layer 2)
  uint32_t* mask;          // layer 2: [B x nrows/32]
  uint32_t* umask;         // layer 2: [nrows/32] union of the batch's rows, or null
  float* logits;           // layer 2: [B x nrows] or null
  float threshold;
  float* part;             // layer 1: [gridDim.y x B x nrows] partial W1 x
  int len, nrows, B;
};

template <bool L1, int DT, int N, int NS>
__global__ void __launch_bounds__(kUmmaThreads, 2)
    k_umma_pred(const __grid_constant__ CUtensorMap tm_b0, const __grid_constant__ CUtensorMap tm_b1,
                UmmaPredParams p) {
  constexpr int NB = L1 ? 1 : 2;  // activation tiles per stage
  constexpr int ABYTES = kUmmaM * kUmmaK * 2;
  constexpr int BBYTES = N * kUmmaK * 2;
  constexpr int STAGE = ABYTES + NB * BBYTES;
  constexpr uint32_t NCOL = N <= 32 ? 32 : N <= 64 ? 64 : N <= 128 ? 128 : 256;
  constexpr uint32_t IDESC = idesc_f16<DT, kUmmaM, N, 0, 0>();
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  __shared__ uint64_t full[NS], empty[NS], done;
  __shared__ uint32_t tmem_base;

  pdl_wait();
  pdl_trigger();
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  const int row0 = blockIdx.x * kUmmaM;
  const int T = p.len / kUmmaK;  // stages of the whole contraction
  const int st0 = (int)(((long long)T * blockIdx.y) / gridDim.y);
  const int nst = (int)(((long long)T * (blockIdx.y + 1)) / gridDim.y) - st0;
  if (t == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1 + kUmmaM);
      mbar_init(&empty[s], 1);
    }
    mbar_init(&done, 1);
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(&tmem_base, NCOL);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;

  if (warp == 0) {
    if (lane == 0) {
      for (int i = 0; i < nst; ++i) {
        const int s = i % NS;
        if (i >= NS && !mbar_wait(&empty[s], ((i / NS) - 1) & 1)) break;
        uint8_t* st = smem + (size_t)s * STAGE;
        mbar_arrive_expect_tx(&full[s], NB * BBYTES);
        tma_load2d(st + ABYTES, &tm_b0, (st0 + i) * kUmmaK, 0, &full[s]);
        if constexpr (!L1) tma_load2d(st + ABYTES + BBYTES, &tm_b1, (st0 + i) * kUmmaK, 0, &full[s]);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      for (int i = 0; i < nst; ++i) {
        const int s = i % NS;
        if (!mbar_wait(&full[s], (i / NS) & 1)) break;
        fence_proxy_async_smem();  // the builders' async copies
        tc_fence_after();
        const uint32_t sa = smem_u32(smem + (size_t)s * STAGE);
        const uint32_t sh = sa + ABYTES, sl = sh + BBYTES;
#pragma unroll
        for (int kk = 0; kk < kUmmaK / 16; ++kk) {
          const uint64_t ad = sw128_desc(sa + 32 * kk, 16, 1024);
          umma_f16(tmem, ad, sw128_desc(sh + 32 * kk, 16, 1024), IDESC, (i | kk) != 0);
          if constexpr (!L1) umma_f16(tmem, ad, sw128_desc(sl + 32 * kk, 16, 1024), IDESC, 1);
        }
        umma_commit(&empty[s]);
      }
      umma_commit(&done);
    }
    __syncwarp();
  } else {
    // thread m copies chunk c = m % 8 of rows 8 (m / 8) + j of each stage
    // straight into the swizzled layout (cp.async; rows past the matrix
    // are zero-filled)
    const int m = t - 64;
    const int c = m & 7, g = m >> 3;
    const size_t rb = (size_t)p.len * 2;
    const uint8_t* rowp[8];
    uint32_t nbytes[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int row = row0 + 8 * g + j;
      nbytes[j] = row < p.nrows ? 16u : 0u;
      rowp[j] = p.w + (size_t)(row < p.nrows ? row : 0) * rb + (size_t)st0 * 128 + (size_t)c * 16;
    }
    // prefetch: thread m asks for row m's 128-byte piece of stage i + kPfAhead
    const bool plive = row0 + m < p.nrows;
    const uint8_t* prow = p.w + (size_t)(plive ? row0 + m : 0) * rb + (size_t)st0 * 128;
    for (int j = 0; j < kPfAhead && j < nst; ++j)
      if (plive) prefetch_line(prow + 128 * j);
    bool ok = true;
    const uint32_t gb = smem_u32(smem + g * 1024);
    const uint64_t pol = policy_evict_first();
    for (int i = 0; i < nst; ++i) {
      const int s = i % NS;
      if (plive && i + kPfAhead < nst) prefetch_line(prow + 128 * (i + kPfAhead));
      if (i >= NS && !mbar_wait(&empty[s], ((i / NS) - 1) & 1)) {
        ok = false;
        break;
      }
      const uint32_t st = gb + (uint32_t)(s * STAGE);
#pragma unroll
      for (int j = 0; j < 8; ++j)
        cp_async16_fill(st + (uint32_t)(j * 128 + ((c ^ j) << 4)), rowp[j] + 128 * i, nbytes[j],
                        pol);
      cp_async_arrive_noinc(&full[s]);
    }
    cp_async_wait_all();
    // epilogue: lane = row 32 (w % 4) + lane of the tile
    const int quad = warp & 3;
    const int n = row0 + quad * 32 + lane;
    const bool done_ok = nst == 0 || mbar_wait_sleep(&done, 0);
    tc_fence_after();
    if constexpr (L1) {
#pragma unroll
      for (int c0 = 0; c0 < N; c0 += 8) {
        uint32_t rr[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
        if (nst > 0) {
          tmem_ld8(tmem + ((uint32_t)(quad * 32) << 16) + c0, rr);
          tmem_wait_ld();
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int b = c0 + j;
          if (b < p.B && n < p.nrows)
            p.part[((size_t)blockIdx.y * p.B + b) * p.nrows + n] =
                (ok && done_ok) ? __uint_as_float(rr[j]) : 0.f;
        }
      }
    } else {
      const float bias = n < p.nrows ? p.bias[n] : 0.f;
      uint32_t uni = 0u;
#pragma unroll
      for (int c0 = 0; c0 < N; c0 += 8) {
        uint32_t rr[8];
        tmem_ld8(tmem + ((uint32_t)(quad * 32) << 16) + c0, rr);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int b = c0 + j;
          if (b < p.B) {  // warp-uniform
            const float sv = __uint_as_float(rr[j]) + bias;
            const bool valid = ok && done_ok && n < p.nrows;
            if (p.logits && valid) p.logits[(size_t)b * p.nrows + n] = sv;
            const uint32_t word = __ballot_sync(0xffffffffu, valid && sv > p.threshold);
            uni |= word;
            if (lane == 0 && row0 + quad * 32 < p.nrows)
              p.mask[(size_t)b * (p.nrows / 32) + (row0 + quad * 32) / 32] = word;
          }
        }
      }
      if (p.umask && lane == 0 && row0 + quad * 32 < p.nrows)
        p.umask[(row0 + quad * 32) / 32] = uni;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, NCOL);
  }
}

// Predictor layer 1 from its split-contraction partials: a = relu(sum over
// the S slices in order + b1), written as fp32 (aout, for the CUDA-core
// layer 2) and/or as the hi + lo 16-bit parts that the tensor-core layer 2
// multiplies (ahi, alo).  part [S x B x r].
template <int DT>
__global__ void __launch_bounds__(256) k_pred1_finish(const float* __restrict__ part, int S, int B,
                                                      int r, const float* __restrict__ b1,
                                                      uint16_t* __restrict__ ahi,
                                                      uint16_t* __restrict__ alo,
                                                      float* __restrict__ aout) {
  pdl_wait();
  pdl_trigger();
  const int e = blockIdx.x * 256 + threadIdx.x;
  if (e >= B * r) return;
  float z = part[e];
  for (int y = 1; y < S; ++y) z += part[(size_t)y * B * r + e];
  if (b1) z += b1[e % r];
  const float a = fmaxf(z, 0.f);
  if (aout) aout[e] = a;
  if (ahi) {
    const uint16_t hi = to16<DT>(a);
    ahi[e] = hi;
    alo[e] = to16<DT>(a - from16<DT>(hi));
  }
}

}  // namespace pi
