// Compaction and the gathered (neuron-aware) FFN.
//
// PowerInfer keeps, per layer, a table that maps each active neuron to its
// original row (unite.ai page, "Neuronen-Platzierung und -Verwaltung"), and
// its neuron-aware operator computes only those neurons' row vectors of W_up
// (and W_gate) and W_down^T, with no sparse-format conversion (same page,
// "Neuronenbewusster Operator").  Here W_down is stored transposed, so a
// neuron's down-projection column is one contiguous row too, and every
// gathered read streams one contiguous row.
#pragma once
#include "pi_predict.cuh"

namespace pi {

// --------------------------------------------------------------- compaction
// One CTA of 1024 threads; thread t owns words [t*WPT, t*WPT + WPT) of the
// OR of the batch's mask rows, so an exclusive scan of the per-thread
// popcounts gives every neuron its position in the ascending list.
constexpr int kCompactThreads = 1024;

__global__ void __launch_bounds__(kCompactThreads, 1)
    k_compact(const uint32_t* __restrict__ mask, int B, int F, int32_t* __restrict__ idx,
              int32_t* __restrict__ count) {
  __shared__ int warp_tot[32];
  pdl_wait();
  pdl_trigger();
  const int W = F / 32;
  const int wpt = (W + kCompactThreads - 1) / kCompactThreads;
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  uint32_t words[2];
  int mine = 0;
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    words[k] = 0u;
    const int w = t * wpt + k;
    if (k < wpt && w < W) {
      uint32_t m = 0u;
      for (int b = 0; b < B; ++b) m |= mask[(size_t)b * W + w];
      words[k] = m;
      mine += __popc(m);
    }
  }
  // block exclusive scan of `mine`
  int incl = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int v = warp_tot[lane];
    int s = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += u;
    }
    warp_tot[lane] = s - v;  // exclusive prefix of warp totals
    if (lane == 31) *count = s;
  }
  __syncthreads();
  int pos = warp_tot[warp] + incl - mine;
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    uint32_t m = words[k];
    const int base = (t * wpt + k) * 32;
    while (m) {
      const int bit = __ffs(m) - 1;
      idx[pos++] = base + bit;
      m &= m - 1;
    }
  }
}

// ------------------------------------------------------ gathered FFN
// Each CTA takes a contiguous, balanced slice [k0, k1) of the K active
// neurons.  The list comes either from the caller (idx, count) or straight
// from the predictor's mask bits: every CTA scans the (batch-OR of the) mask
// words itself, so the index list never round-trips through another kernel;
// the CTA stages its slice of neuron ids and their biases in shared memory.
// Each CTA writes its partial y to part[cta]; k_reduce sums the partials in a
// fixed order (no atomics: y is bit-reproducible).
struct FfnParams {
  const uint8_t* w_act;    // W_up (ReLU) or W_gate (ReGLU)
  const uint8_t* w_up;     // W_up (ReGLU only)
  const uint8_t* w_dn;     // W_down^T
  const float* b_act;      // b_up (ReLU) / b_gate (ReGLU), or null
  const uint16_t* x;       // [B x d]
  const int32_t* idx;      // explicit neuron list (when mask is null)
  const int32_t* count;
  const uint32_t* mask;    // [mask_rows x F/32] predicted bits, or null
  int mask_rows;
  int32_t* idx_out;        // mask mode: the ascending list is written here, or null
  int32_t* count_out;
  float* part;             // [gridDim.x x B x d]
  int d, F;
  uint32_t row_bytes;
  int list_cap;
  // weights the next kernels will read (the next layer's predictor), asked
  // of the L2 while this kernel's prologue leaves DRAM idle; null for none
  const uint8_t* pf_base[2];
  size_t pf_bytes[2];
};

// Block-wide exclusive scan of one int per thread (all NT threads of the CTA).
template <int NT>
__device__ __forceinline__ int block_excl_scan(int v, int* scratch /* >= 33 ints */, int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int u = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += u;
  }
  if (lane == 31) scratch[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int t = lane < NT / 32 ? scratch[lane] : 0;
    int s = t;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += u;
    }
    scratch[lane] = s - t;
    if (lane == 31) scratch[32] = s;
  }
  __syncthreads();
  total = scratch[32];
  return scratch[warp] + incl - v;
}

// This CTA's slice [k0, k1) of the neuron list, staged in ids / lbias (ids
// of invalid explicit entries are -1).  All NT threads call it; it ends with a
// CTA barrier.
template <int NT, bool BIAS = true>
__device__ void build_slice(const FfnParams& p, int* scratch, uint32_t* wbuf /* [2 x F/32] */,
                            int* ids, float* lbias, int& k0, int& k1) {
  const int G = gridDim.x;
  if (p.mask) {
    const int W = p.F / 32;
    const int wpt = (W + NT - 1) / NT;
    const int w0 = threadIdx.x * wpt;
    uint32_t words[8];
    int mine = 0;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      words[k] = 0u;
      if (k < wpt && w0 + k < W) {
        uint32_t m = 0u;
        for (int b = 0; b < p.mask_rows; ++b) m |= p.mask[(size_t)b * W + w0 + k];
        words[k] = m;
        mine += __popc(m);
      }
    }
    int K;
    int pos = block_excl_scan<NT>(mine, scratch, K);
    k0 = (int)(((long long)K * blockIdx.x) / G);
    k1 = (int)(((long long)K * (blockIdx.x + 1)) / G);
    if (blockIdx.x == 0 && threadIdx.x == 0 && p.count_out) *p.count_out = K;
    // per-word exclusive prefix counts and the words themselves ...
    uint32_t* wmask = wbuf;
    int* wpre = reinterpret_cast<int*>(wbuf + W);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      if (k < wpt && w0 + k < W) {
        wmask[w0 + k] = words[k];
        wpre[w0 + k] = pos;
        pos += __popc(words[k]);
      }
    }
    __syncthreads();
    // ... so that slice position i (rank k0 + i of the union) is found in
    // parallel: its word by binary search, then its bit within the word
    for (int i = threadIdx.x; i < k1 - k0; i += NT) {
      const int q = k0 + i;
      int lo = 0, hi = W - 1;  // the last word whose prefix is <= q
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (wpre[mid] <= q) lo = mid;
        else hi = mid - 1;
      }
      const int nid = lo * 32 + (int)__fns(wmask[lo], 0, q - wpre[lo] + 1);
      ids[i] = nid;
      if (BIAS) lbias[i] = p.b_act ? p.b_act[nid] : 0.f;
      if (p.idx_out) p.idx_out[q] = nid;
    }
  } else {
    int K = *p.count;
    K = K < 0 ? 0 : (K > p.F ? p.F : K);
    k0 = (int)(((long long)K * blockIdx.x) / G);
    k1 = (int)(((long long)K * (blockIdx.x + 1)) / G);
    for (int i = threadIdx.x; i < k1 - k0; i += NT) {
      const int nid = p.idx[k0 + i];
      const bool valid = nid >= 0 && nid < p.F;
      if (!valid) set_error(kErrBadIndex);
      ids[i] = valid ? nid : -1;
      if (BIAS) lbias[i] = (valid && p.b_act) ? p.b_act[nid] : 0.f;
    }
  }
  __syncthreads();
}


// ------------------------------------------ gathered FFN, 16-bit weights
// Two phases per CTA over its slice of the neuron list:
//   up:   the whole CTA works on every neuron, a group of R neurons at a time:
//         thread t holds the 16-byte chunks t, t+NT, ... of x (fp32, in
//         registers) and loads the same chunks of each of the group's rows
//         with 128-bit loads straight into registers, so every row is
//         requested whole and at once.  One block reduction per group gives
//         the group's h, stored in shared memory;
//   down: after one CTA barrier, thread t owns the 16-byte column chunks
//         t, t+NT, ... of y and streams those chunks of every neuron's
//         W_down^T row through registers, accumulating h * row in fp32.
// Both phases are software-pipelined over two register buffers, so the next
// group's loads are always in flight while the current one is consumed, and
// the first loads of each phase are issued before the barrier that precedes
// it.  Every gathered row is read exactly once.
// (Measured on B200: gathered 8 KB rows stream at about 6.1 TB/s through
// registers; a shared-memory ring fed by one bulk-copy thread per CTA reached
// about 5.4 TB/s with no work attached, and L2 prefetching of the rows ahead
// of use made this kernel slower.)
#ifndef PI_LDG_THREADS
#define PI_LDG_THREADS 256
#endif
#ifndef PI_UP_REGS
#define PI_UP_REGS 8
#endif
#ifndef PI_DOWN_REGS
#define PI_DOWN_REGS 8
#endif
constexpr int kLdgThreads = PI_LDG_THREADS;
constexpr int kLdgWarps = kLdgThreads / 32;
constexpr int kUpRegs = PI_UP_REGS;      // up phase: 16-byte loads per thread per buffer
constexpr int kDownRegs = PI_DOWN_REGS;  // down phase: 16-byte loads per thread per buffer

// WDT: 0 fp16, 1 bf16 (activations of the same type).  ACT: 0 ReLU, 1 ReGLU,
// 2 Squared-ReLU.  CPT: column chunks per thread.  CPS: CTAs per SM.
template <int WDT, int ACT, int B, int CPT, int CPS>
__global__ void __launch_bounds__(kLdgThreads, CPS) k_ffn_ldg(FfnParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr int NUP = ACT == 1 ? 2 : 1;  // rows per neuron in the up phase
  constexpr int R = kUpRegs / (NUP * CPT) > 0 ? kUpRegs / (NUP * CPT) : 1;  // neurons per group
  constexpr int VG = R * NUP * B;        // dot products per group
  constexpr int SHG = 5 - log2c<VG>();
  static_assert(VG <= 32 && (VG & (VG - 1)) == 0, "a group's dot products fit one warp reduction");
  constexpr int DH = kDownRegs / CPT > 0 ? kDownRegs / CPT : 1;  // down: neurons per buffer
  int* scratch = reinterpret_cast<int*>(smem);                 // 64 ints
  int* ids = reinterpret_cast<int*>(smem + 256);               // [list_cap]
  float* lbias = reinterpret_cast<float*>(ids + p.list_cap);   // [list_cap]
  float* hs = lbias + p.list_cap;                              // [list_cap * B]
  uint32_t* wbuf = reinterpret_cast<uint32_t*>(hs + (size_t)p.list_cap * B);  // [2 x F/32]
  __shared__ float red[2][kLdgWarps][VG];

  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int d = p.d, nchunks = d / 8;
  const size_t rb = (size_t)d * 2;
  // gathered rows are read once: first in line for eviction from the L2, so
  // that the prefetched weights below stay there
  const uint64_t pol = policy_evict_first();
#ifndef PI_FFN_PF
#define PI_FFN_PF 1
#endif
  if (PI_FFN_PF && t == 0) {
    prefetch_l2_share(p.pf_base[0], p.pf_bytes[0], blockIdx.x, gridDim.x);
    prefetch_l2_share(p.pf_base[1], p.pf_bytes[1], blockIdx.x, gridDim.x);
  }

  pdl_trigger();
  pdl_wait();  // the list (or mask) and x come from earlier kernels
  // this thread's chunks of x, requested together with the mask words
  uint4 xq[B][CPT];
#pragma unroll
  for (int b = 0; b < B; ++b)
#pragma unroll
    for (int c = 0; c < CPT; ++c) {
      const int u = t + kLdgThreads * c;
      xq[b][c] = u < nchunks ? reinterpret_cast<const uint4*>(p.x + (size_t)b * d)[u]
                             : make_uint4(0, 0, 0, 0);
    }
  int k0, k1;
  build_slice<kLdgThreads, false>(p, scratch, wbuf, ids, lbias, k0, k1);
  const int n = k1 - k0;

  // ------------------------------------------------------------- up phase
  const int ngroups = (n + R - 1) / R;
  auto load_up = [&](int g, uint4 (&r)[R][NUP][CPT]) {
#pragma unroll
    for (int j = 0; j < R; ++j) {
      const int i = g * R + j;
      const int nid = i < n ? ids[i] : -1;
#pragma unroll
      for (int m = 0; m < NUP; ++m) {
        const uint8_t* row = (m == 0 ? p.w_act : p.w_up) + (size_t)(nid < 0 ? 0 : nid) * rb;
#pragma unroll
        for (int c = 0; c < CPT; ++c) {
          const int u = t + kLdgThreads * c;
          r[j][m][c] = (nid >= 0 && u < nchunks) ? ldg_stream_hint(row + (size_t)u * 16, pol)
                                                 : make_uint4(0, 0, 0, 0);
        }
      }
    }
  };
  uint4 ua[R][NUP][CPT], ub[R][NUP][CPT];
  if (ngroups > 0) load_up(0, ua);
  // biases of the slice: read only after the first group's barrier
  for (int i = t; i < n; i += kLdgThreads)
    lbias[i] = (p.b_act && ids[i] >= 0) ? p.b_act[ids[i]] : 0.f;
  float xr[B][CPT][8];
#pragma unroll
  for (int b = 0; b < B; ++b)
#pragma unroll
    for (int c = 0; c < CPT; ++c) widen8<WDT>(xq[b][c], xr[b][c]);

  auto consume_up = [&](int g, const uint4 (&r)[R][NUP][CPT]) {
    float v[VG];
#pragma unroll
    for (int j = 0; j < R; ++j)
#pragma unroll
      for (int m = 0; m < NUP; ++m)
#pragma unroll
        for (int b = 0; b < B; ++b) {
          float z = 0.f;
#pragma unroll
          for (int c = 0; c < CPT; ++c) z += dot8<WDT>(r[j][m][c], xr[b][c]);
          v[(j * NUP + m) * B + b] = z;
        }
    const float tot = warp_reduce_transposed<VG>(v);
    const int buf = g & 1;
    if ((lane & ((1 << SHG) - 1)) == 0) red[buf][warp][lane >> SHG] = tot;
    __syncthreads();
    if (t < R * B) {
      const int j = t / B, b = t % B, i = g * R + j;
      if (i < n) {
        float act = 0.f, up = 1.f;
#pragma unroll
        for (int w = 0; w < kLdgWarps; ++w) act += red[buf][w][(j * NUP) * B + b];
        if constexpr (ACT == 1) {
          up = 0.f;
#pragma unroll
          for (int w = 0; w < kLdgWarps; ++w) up += red[buf][w][(j * NUP + 1) * B + b];
        }
        const float r = fmaxf(act + lbias[i], 0.f);
        const float h = ACT == 2 ? r * r : r * up;
        hs[(size_t)i * B + b] = ids[i] < 0 ? 0.f : h;
      }
    }
  };

  for (int g = 0; g < ngroups; g += 2) {
    if (g + 1 < ngroups) load_up(g + 1, ub);
    consume_up(g, ua);
    if (g + 1 < ngroups) {
      if (g + 2 < ngroups) load_up(g + 2, ua);
      consume_up(g + 1, ub);
    }
  }

  // ----------------------------------------------------------- down phase
  auto load_down = [&](int i0, uint4 (&r)[DH][CPT]) {
#pragma unroll
    for (int j = 0; j < DH; ++j) {
      const int i = i0 + j;
      const int nid = (i < n && ids[i] >= 0) ? ids[i] : 0;
      const uint8_t* row = p.w_dn + (size_t)nid * rb;
#pragma unroll
      for (int c = 0; c < CPT; ++c) {
        const int u = t + kLdgThreads * c;
        r[j][c] = (i < n && u < nchunks) ? ldg_stream_hint(row + (size_t)u * 16, pol)
                                         : make_uint4(0, 0, 0, 0);
      }
    }
  };
  float acc[B][CPT][8];
#pragma unroll
  for (int b = 0; b < B; ++b)
#pragma unroll
    for (int c = 0; c < CPT; ++c)
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[b][c][e] = 0.f;
  auto fma_down = [&](int i0, const uint4 (&r)[DH][CPT]) {
#pragma unroll
    for (int j = 0; j < DH; ++j) {
      const int i = i0 + j;
      if (i < n) {
        float hb[B];
#pragma unroll
        for (int b = 0; b < B; ++b) hb[b] = hs[(size_t)i * B + b];
#pragma unroll
        for (int c = 0; c < CPT; ++c) {
          const uint32_t wv[4] = {r[j][c].x, r[j][c].y, r[j][c].z, r[j][c].w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = unpack2<WDT>(wv[e]);
#pragma unroll
            for (int b = 0; b < B; ++b) {
              acc[b][c][2 * e] = fmaf(hb[b], f.x, acc[b][c][2 * e]);
              acc[b][c][2 * e + 1] = fmaf(hb[b], f.y, acc[b][c][2 * e + 1]);
            }
          }
        }
      }
    }
  };

  uint4 d0[DH][CPT], d1[DH][CPT];
  load_down(0, d0);  // in flight across the barrier (rows need no h)
  __syncthreads();   // every h of the slice is in shared memory
  for (int i0 = 0; i0 < n; i0 += 2 * DH) {
    load_down(i0 + DH, d1);
    fma_down(i0, d0);
    if (i0 + DH < n) {
      load_down(i0 + 2 * DH, d0);
      fma_down(i0 + DH, d1);
    }
  }

  // partial y of this CTA
#pragma unroll
  for (int b = 0; b < B; ++b)
#pragma unroll
    for (int c = 0; c < CPT; ++c) {
      const int u = t + kLdgThreads * c;
      if (u < nchunks) {
        float4* dst = reinterpret_cast<float4*>(p.part + ((size_t)blockIdx.x * B + b) * d +
                                                (size_t)u * 8);
        dst[0] = make_float4(acc[b][c][0], acc[b][c][1], acc[b][c][2], acc[b][c][3]);
        dst[1] = make_float4(acc[b][c][4], acc[b][c][5], acc[b][c][6], acc[b][c][7]);
      }
    }
}

// ------------------------------------------------ gathered FFN, Q4_0 (LDG)
// Q4_0 rows (d/32 blocks of 18 bytes: fp16 scale, then 16 bytes whose byte j
// holds element j in its low nibble and element j+16 in its high nibble) are
// streamed through registers like the 16-bit rows.  Thread t owns block t of
// every row: its 32 elements of x (fp32, in registers) in the up phase and its
// 32 columns of y in the down phase.  The 32 blocks of warp w form one
// 16-byte aligned 576-byte span (36 chunks), which the warp loads with
// 128-bit loads and passes through a 576-byte shared-memory slot so that each
// lane reads back its own 18 bytes.  Each nibble q becomes the exact float
// f = 1 + q/16 with one byte permute (exponent byte 0x3F, mantissa byte
// 0x80 | 8q, prepared four at a time), so a block's dot product is
//   scale * sum_e (q_e - 8) x_e = scale * (16 sum_e f_e x_e - 24 sum_e x_e)
// and the down phase adds (16 h scale) f_e per column and -24 h scale once.
#ifndef PI_Q4_SPANS
#define PI_Q4_SPANS 4
#endif
constexpr int kQ4Threads = 256;
constexpr int kQ4Warps = kQ4Threads / 32;
constexpr int kQ4Spans = PI_Q4_SPANS;  // rows in flight per thread per buffer
constexpr int kQ4SpanBytes = 576;      // 32 blocks x 18 bytes

// This lane's block out of its warp's span in shared memory (144 words).
__device__ __forceinline__ void q4_lane_block(const uint32_t* span, int lane, uint32_t& sc,
                                              uint32_t (&q)[4]) {
  const int w0 = (9 * lane) >> 1;  // word holding byte 18 * lane
  uint32_t w[5];
#pragma unroll
  for (int k = 0; k < 5; ++k) w[k] = span[w0 + k];
  const bool odd = lane & 1;  // odd lanes start 2 bytes into the word
  sc = odd ? (w[0] >> 16) : (w[0] & 0xffffu);
#pragma unroll
  for (int k = 0; k < 4; ++k) q[k] = odd ? w[k + 1] : __funnelshift_r(w[k], w[k + 1], 16);
}

// The four low (hi = false) or high nibbles of w, each as the byte 0x80 | 8q.
__device__ __forceinline__ uint32_t nib_bytes(uint32_t w, bool hi) {
  return ((hi ? (w >> 1) : (w << 3)) & 0x78787878u) | 0x80808080u;
}
// 1 + q/16 for the nibble in byte i of v (from nib_bytes): bits 0x3F800000 | q << 19.
__device__ __forceinline__ float nib16(uint32_t v, int i) {
  return __uint_as_float(__byte_perm(v, 0x3F000000u, 0x7044u | ((uint32_t)i << 8)));
}

template <int ACT, int B>
__global__ void __launch_bounds__(kQ4Threads, B == 1 ? 2 : 1) k_ffn_q4(FfnParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr int NUP = ACT == 1 ? 2 : 1;                 // up-phase rows per neuron
  constexpr int R = kQ4Spans / NUP > 0 ? kQ4Spans / NUP : 1;  // neurons per up group
  constexpr int VG = R * NUP * B;
  constexpr int SHG = 5 - log2c<VG>();
  static_assert(VG <= 32 && (VG & (VG - 1)) == 0, "a group's dot products fit one warp reduction");
  constexpr int DH = kQ4Spans;                          // down: neurons per buffer
  int* scratch = reinterpret_cast<int*>(smem);
  int* ids = reinterpret_cast<int*>(smem + 256);
  float* lbias = reinterpret_cast<float*>(ids + p.list_cap);
  float* hs = lbias + p.list_cap;
  uint32_t* wbuf = reinterpret_cast<uint32_t*>(hs + (size_t)p.list_cap * B);
  __shared__ __align__(16) uint32_t spans[kQ4Warps][kQ4SpanBytes / 4];
  __shared__ float red[2][kQ4Warps][VG];

  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int d = p.d, nb = d / 32;
  const size_t rb = (size_t)nb * 18;
  const bool mine = t < nb;                              // this thread owns block t
  const int nv = min(32, max(0, nb - 32 * warp));        // blocks in this warp's span
  const int cnt = nv * 9 / 8;                            // 16-byte chunks in the span
  const uint64_t pol = policy_evict_first();
  if (t == 0) {
    prefetch_l2_share(p.pf_base[0], p.pf_bytes[0], blockIdx.x, gridDim.x);
    prefetch_l2_share(p.pf_base[1], p.pf_bytes[1], blockIdx.x, gridDim.x);
  }

  pdl_trigger();
  pdl_wait();  // the list (or mask) and x come from earlier kernels
  uint4 xq[B][4];
#pragma unroll
  for (int b = 0; b < B; ++b)
#pragma unroll
    for (int k = 0; k < 4; ++k)
      xq[b][k] = mine ? reinterpret_cast<const uint4*>(p.x + (size_t)b * d + (size_t)t * 32)[k]
                      : make_uint4(0, 0, 0, 0);
  int k0, k1;
  build_slice<kQ4Threads, false>(p, scratch, wbuf, ids, lbias, k0, k1);
  const int n = k1 - k0;

  struct Span { uint4 m, e; };
  auto load_span = [&](const uint8_t* row, Span& sp) {
    const uint4* src = reinterpret_cast<const uint4*>(row + (size_t)warp * kQ4SpanBytes);
    sp.m = lane < cnt ? ldg_stream_hint(src + lane, pol) : make_uint4(0, 0, 0, 0);
    sp.e = lane + 32 < cnt ? ldg_stream_hint(src + 32 + lane, pol) : make_uint4(0, 0, 0, 0);
  };
  // pass a span through the warp's slot; returns this lane's scale and nibbles
  auto open_span = [&](const Span& sp, float& scale, uint32_t (&q)[4]) {
    uint4* slot = reinterpret_cast<uint4*>(spans[warp]);
    __syncwarp();
    if (lane < cnt) slot[lane] = sp.m;
    if (lane + 32 < cnt) slot[32 + lane] = sp.e;
    __syncwarp();
    uint32_t sc;
    q4_lane_block(spans[warp], lane, sc, q);
    scale = __half2float(__ushort_as_half((unsigned short)sc));
  };

  // ------------------------------------------------------------- up phase
  const int ngroups = (n + R - 1) / R;
  auto load_up = [&](int g, Span (&r)[R][NUP]) {
#pragma unroll
    for (int j = 0; j < R; ++j) {
      const int i = g * R + j;
      const int nid = i < n ? ids[i] : -1;
#pragma unroll
      for (int m = 0; m < NUP; ++m) {
        if (nid >= 0) {
          load_span((m == 0 ? p.w_act : p.w_up) + (size_t)nid * rb, r[j][m]);
        } else {
          r[j][m].m = make_uint4(0, 0, 0, 0);
          r[j][m].e = make_uint4(0, 0, 0, 0);
        }
      }
    }
  };
  Span ua[R][NUP], ub[R][NUP];
  if (ngroups > 0) load_up(0, ua);
  for (int i = t; i < n; i += kQ4Threads)
    lbias[i] = (p.b_act && ids[i] >= 0) ? p.b_act[ids[i]] : 0.f;
  float xr[B][32], sx[B];
#pragma unroll
  for (int b = 0; b < B; ++b) {
    float s8 = 0.f;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      widen8<0>(xq[b][k], xr[b] + 8 * k);
#pragma unroll
      for (int e = 0; e < 8; ++e) s8 += xr[b][8 * k + e];
    }
    sx[b] = s8;
  }

  auto consume_up = [&](int g, const Span (&r)[R][NUP]) {
    float v[VG];
#pragma unroll
    for (int j = 0; j < R; ++j)
#pragma unroll
      for (int m = 0; m < NUP; ++m) {
        float scale;
        uint32_t q[4];
        open_span(r[j][m], scale, q);
        float dq[B];
#pragma unroll
        for (int b = 0; b < B; ++b) dq[b] = 0.f;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint32_t L = nib_bytes(q[k], false), H = nib_bytes(q[k], true);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float fl = nib16(L, i), fh = nib16(H, i);
#pragma unroll
            for (int b = 0; b < B; ++b) {
              dq[b] = fmaf(fl, xr[b][4 * k + i], dq[b]);
              dq[b] = fmaf(fh, xr[b][4 * k + i + 16], dq[b]);
            }
          }
        }
#pragma unroll
        for (int b = 0; b < B; ++b)
          v[(j * NUP + m) * B + b] = mine ? scale * fmaf(16.f, dq[b], -24.f * sx[b]) : 0.f;
      }
    const float tot = warp_reduce_transposed<VG>(v);
    const int buf = g & 1;
    if ((lane & ((1 << SHG) - 1)) == 0) red[buf][warp][lane >> SHG] = tot;
    __syncthreads();
    if (t < R * B) {
      const int j = t / B, b = t % B, i = g * R + j;
      if (i < n) {
        float act = 0.f, up = 1.f;
#pragma unroll
        for (int w = 0; w < kQ4Warps; ++w) act += red[buf][w][(j * NUP) * B + b];
        if constexpr (ACT == 1) {
          up = 0.f;
#pragma unroll
          for (int w = 0; w < kQ4Warps; ++w) up += red[buf][w][(j * NUP + 1) * B + b];
        }
        const float rr = fmaxf(act + lbias[i], 0.f);
        const float h = ACT == 2 ? rr * rr : rr * up;
        hs[(size_t)i * B + b] = ids[i] < 0 ? 0.f : h;
      }
    }
  };

  for (int g = 0; g < ngroups; g += 2) {
    if (g + 1 < ngroups) load_up(g + 1, ub);
    consume_up(g, ua);
    if (g + 1 < ngroups) {
      if (g + 2 < ngroups) load_up(g + 2, ua);
      consume_up(g + 1, ub);
    }
  }

  // ----------------------------------------------------------- down phase
  auto load_down = [&](int i0, Span (&r)[DH]) {
#pragma unroll
    for (int j = 0; j < DH; ++j) {
      const int i = i0 + j;
      if (i < n && ids[i] >= 0) {
        load_span(p.w_dn + (size_t)ids[i] * rb, r[j]);
      } else {
        r[j].m = make_uint4(0, 0, 0, 0);
        r[j].e = make_uint4(0, 0, 0, 0);
      }
    }
  };
  float acc[B][32], cst[B];
#pragma unroll
  for (int b = 0; b < B; ++b) {
    cst[b] = 0.f;
#pragma unroll
    for (int e = 0; e < 32; ++e) acc[b][e] = 0.f;
  }
  auto fma_down = [&](int i0, const Span (&r)[DH]) {
#pragma unroll
    for (int j = 0; j < DH; ++j) {
      const int i = i0 + j;
      if (i < n) {  // CTA-uniform: every lane takes part in the span exchange
        float scale;
        uint32_t q[4];
        open_span(r[j], scale, q);
        float hsc[B];
#pragma unroll
        for (int b = 0; b < B; ++b) {
          const float hq = hs[(size_t)i * B + b] * scale;  // h * scale
          hsc[b] = 16.f * hq;
          cst[b] = fmaf(-24.f, hq, cst[b]);
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint32_t L = nib_bytes(q[k], false), H = nib_bytes(q[k], true);
#pragma unroll
          for (int ii = 0; ii < 4; ++ii) {
            const float fl = nib16(L, ii), fh = nib16(H, ii);
#pragma unroll
            for (int b = 0; b < B; ++b) {
              acc[b][4 * k + ii] = fmaf(hsc[b], fl, acc[b][4 * k + ii]);
              acc[b][4 * k + ii + 16] = fmaf(hsc[b], fh, acc[b][4 * k + ii + 16]);
            }
          }
        }
      }
    }
  };

  Span d0[DH], d1[DH];
  load_down(0, d0);  // in flight across the barrier (rows need no h)
  __syncthreads();   // every h of the slice is in shared memory
  for (int i0 = 0; i0 < n; i0 += 2 * DH) {
    load_down(i0 + DH, d1);
    fma_down(i0, d0);
    if (i0 + DH < n) {
      load_down(i0 + 2 * DH, d0);
      fma_down(i0 + DH, d1);
    }
  }

  // partial y of this CTA: columns 32t .. 32t+31
  if (mine) {
#pragma unroll
    for (int b = 0; b < B; ++b) {
      float4* dst = reinterpret_cast<float4*>(p.part + ((size_t)blockIdx.x * B + b) * d +
                                              (size_t)t * 32);
#pragma unroll
      for (int e = 0; e < 8; ++e)
        dst[e] = make_float4(acc[b][4 * e] + cst[b], acc[b][4 * e + 1] + cst[b],
                             acc[b][4 * e + 2] + cst[b], acc[b][4 * e + 3] + cst[b]);
    }
  }
}

// ------------------------------------------------------ row permutation
// dst row i = src row perm[i] (rows of row_bytes bytes, V-byte units: 16 when
// row_bytes % 16 == 0, else 4).  Grid-stride over (row, unit) pairs, so
// consecutive threads copy consecutive units of one row.  Ids outside
// [0, n) are flagged and their destination rows left untouched.
template <int V>
__global__ void __launch_bounds__(256) k_gather_rows(const uint8_t* __restrict__ src,
                                                     uint8_t* __restrict__ dst,
                                                     const int32_t* __restrict__ perm, int n,
                                                     int row_units) {
  pdl_wait();
  pdl_trigger();
  const long long total = (long long)n * row_units;
  for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < total;
       e += (long long)gridDim.x * blockDim.x) {
    const int i = (int)(e / row_units), u = (int)(e % row_units);
    const int j = perm[i];
    if (j < 0 || j >= n) {
      if (u == 0) set_error(kErrBadIndex);
      continue;
    }
    if constexpr (V == 16) {
      reinterpret_cast<uint4*>(dst)[e] =
          ldg_stream(src + ((size_t)j * row_units + u) * 16);
    } else {
      reinterpret_cast<uint32_t*>(dst)[e] =
          reinterpret_cast<const uint32_t*>(src)[(size_t)j * row_units + u];
    }
  }
}

// ------------------------------------------------------ partial reduction
// out[i] = sum over g = 0..G-1 of part[g][i], MODE 0 writes y, MODE 1 adds into
// the residual stream.  n4 = number of float4 columns (B*d/4).  A CTA covers 8
// float4 columns with 32 slices each; slice s adds partials g = s, s+32, ...
// in increasing g, and the 32 slice sums are then added in slice order, so the
// summation order is fixed and y is reproducible.
#ifndef PI_RED_COLS
#define PI_RED_COLS 4
#endif
constexpr int kRedCols = PI_RED_COLS;
constexpr int kRedSlices = 256 / kRedCols;

template <int MODE>
__global__ void __launch_bounds__(kRedCols * kRedSlices) k_reduce(const float* __restrict__ part,
                                                                  int G, int n4,
                                                                  float* __restrict__ out) {
  __shared__ float4 sm[kRedSlices][kRedCols];
  pdl_wait();
  pdl_trigger();
  const int cl = threadIdx.x % kRedCols;
  const int sl = threadIdx.x / kRedCols;
  const int col = blockIdx.x * kRedCols + cl;
  float4 t = make_float4(0.f, 0.f, 0.f, 0.f);
  if (col < n4) {
    const float4* src = reinterpret_cast<const float4*>(part);
    int g = sl;
    for (; g + 3 * kRedSlices < G; g += 4 * kRedSlices) {
      const float4 v0 = src[(size_t)g * n4 + col];
      const float4 v1 = src[(size_t)(g + kRedSlices) * n4 + col];
      const float4 v2 = src[(size_t)(g + 2 * kRedSlices) * n4 + col];
      const float4 v3 = src[(size_t)(g + 3 * kRedSlices) * n4 + col];
      t.x += v0.x; t.y += v0.y; t.z += v0.z; t.w += v0.w;
      t.x += v1.x; t.y += v1.y; t.z += v1.z; t.w += v1.w;
      t.x += v2.x; t.y += v2.y; t.z += v2.z; t.w += v2.w;
      t.x += v3.x; t.y += v3.y; t.z += v3.z; t.w += v3.w;
    }
    for (; g < G; g += kRedSlices) {
      const float4 v = src[(size_t)g * n4 + col];
      t.x += v.x; t.y += v.y; t.z += v.z; t.w += v.w;
    }
  }
  sm[sl][cl] = t;
  __syncthreads();
  if (sl == 0 && col < n4) {
    float4 r = sm[0][cl];
#pragma unroll
    for (int k = 1; k < kRedSlices; ++k) {
      const float4 v = sm[k][cl];
      r.x += v.x; r.y += v.y; r.z += v.z; r.w += v.w;
    }
    float4* o = reinterpret_cast<float4*>(out) + col;
    if (MODE == 1) {
      const float4 x = *o;
      r.x += x.x; r.y += x.y; r.z += x.z; r.w += x.w;
    }
    *o = r;
  }
}

// The same sum for a few partial planes (G small, as from the tensor-core
// down projection): one thread per float4 column adds the G planes in order.
template <int MODE>
__global__ void __launch_bounds__(256) k_reduce_few(const float* __restrict__ part, int G, int n4,
                                                    float* __restrict__ out) {
  pdl_wait();
  pdl_trigger();
  const int col = blockIdx.x * 256 + threadIdx.x;
  if (col >= n4) return;
  const float4* src = reinterpret_cast<const float4*>(part);
  float4 t = src[col];
  for (int g = 1; g < G; ++g) {
    const float4 v = src[(size_t)g * n4 + col];
    t.x += v.x; t.y += v.y; t.z += v.z; t.w += v.w;
  }
  float4* o = reinterpret_cast<float4*>(out) + col;
  if (MODE == 1) {
    const float4 x = *o;
    t.x += x.x; t.y += x.y; t.z += x.z; t.w += x.w;
  }
  *o = t;
}

}  // namespace pi
