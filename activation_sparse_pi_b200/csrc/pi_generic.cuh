// Batched kernels for shapes outside the fused kernels' register budget
// (larger batches, e.g. the union-mask batches of 8, 32 and 64 tokens).
// They compute the same steps as the fused path: warp-per-row GEMVs for the
// predictor and the gathered up/gate rows, and a 2-D split (neuron slice x
// column slice) of the gathered down projection with per-slice partials that
// k_reduce sums in a fixed order.
#pragma once
#include "pi_ffn.cuh"

namespace pi {

// ------------------------------------------------------ residual -> x_l
// Same summation order as the fused predictor's rms_cast_to_smem.
template <int DT>
__global__ void __launch_bounds__(256) k_cast_rms(const float* __restrict__ xr,
                                                  uint16_t* __restrict__ xo, int d) {
  __shared__ float red[8];
  pdl_wait();
  pdl_trigger();
  const int b = blockIdx.x, t = threadIdx.x, lane = t & 31, w = t >> 5;
  const float* x = xr + (size_t)b * d;
  float s = 0.f;
  for (int j = t; j < d; j += 256) s = fmaf(x[j], x[j], s);
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane == 0) red[w] = s;
  __syncthreads();
  float tot = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) tot += red[i];
  const float rms = sqrtf(tot / (float)d + kRmsEps);
  for (int j = t; j < d; j += 256) xo[(size_t)b * d + j] = round16<DT>(x[j] / rms);
}

// ------------------------------------------------ warp-per-row batched GEMV
enum { kModePred1 = 0, kModePred2 = 1, kModeUp = 2 };

struct RowsParams {
  const uint8_t* w;        // rows: W1, W2, or the activation rows (W_up / W_gate)
  const uint8_t* w2nd;     // W_up rows for ReGLU (MODE kModeUp)
  const float* bias;       // b1 / b2 / b_act, or null
  const uint16_t* x16;     // [B x len] 16-bit vector (pred1, up)
  const float* x32;        // [B x len] fp32 vector (pred2)
  const int32_t* idx;      // gathered rows (up)
  const int32_t* count;
  float* out;              // a [B x r] | logits [B x F] (nullable) | h [K x B]
  float* part;             // pred1 split over the contraction (gridDim.y > 1):
                           //   [gridDim.y x B x r] raw sums, finished by k_pred1_finish
  uint32_t* mask;          // [B x F/32] (pred2)
  float threshold;
  int nrows;               // r | F | F (bound on K)
  int len;                 // elements per row
  int B;
};

// Dot of one 16-bit row chunk (8 elements) with vector chunks of BB tokens.
template <int MODE, int WDT, int ACT, int BB>
__global__ void __launch_bounds__(256) k_rows(RowsParams p) {
  constexpr int NUP = (MODE == kModeUp && ACT == 1) ? 2 : 1;
  constexpr int XDT = WDT == 1 ? 1 : 0;
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int nw = (gridDim.x * blockDim.x) >> 5;
  int nrows = p.nrows;
  if (MODE == kModeUp) {
    int K = *p.count;
    nrows = K < 0 ? 0 : (K > p.nrows ? p.nrows : K);
  }
  const int B = p.B;
  const size_t rb = WDT == 2 ? (size_t)p.len / 32 * 18 : (size_t)p.len * 2;

  for (int row = gw; row < nrows; row += nw) {
    int nid = row;
    bool valid = true;
    if (MODE == kModeUp) {
      nid = p.idx[row];
      valid = nid >= 0 && nid < p.nrows;
      if (!valid) {
        if (lane == 0) set_error(kErrBadIndex);
        nid = 0;
      }
    }
    float acc[NUP][BB];
#pragma unroll
    for (int m = 0; m < NUP; ++m)
#pragma unroll
      for (int b = 0; b < BB; ++b) acc[m][b] = 0.f;

    if constexpr (WDT == 2) {
#pragma unroll
      for (int m = 0; m < NUP; ++m) {
        const uint8_t* rowp = (m == 0 ? p.w : p.w2nd) + (size_t)nid * rb;
        for (int blk = lane; blk < p.len / 32; blk += 32) {
          const uint16_t* h16 = reinterpret_cast<const uint16_t*>(rowp + (size_t)blk * 18);
          const float sc = __half2float(__ushort_as_half(h16[0]));
          float wv[32];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const uint32_t two = h16[1 + e];  // bytes 2e, 2e+1 of the nibble array
#pragma unroll
            for (int k = 0; k < 2; ++k) {
              const uint32_t byte = (two >> (8 * k)) & 0xffu;
              wv[2 * e + k] = q4_val(byte & 15u) * sc;
              wv[2 * e + k + 16] = q4_val(byte >> 4) * sc;
            }
          }
#pragma unroll
          for (int b = 0; b < BB; ++b) {
            if (b < B) {
              const uint4* xp = reinterpret_cast<const uint4*>(p.x16 + (size_t)b * p.len + blk * 32);
              float s0 = 0.f;
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const uint4 xv = __ldg(xp + q);
                const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  const float2 f = unpack2<0>(xw[e]);
                  s0 = fmaf(wv[q * 8 + 2 * e], f.x, s0);
                  s0 = fmaf(wv[q * 8 + 2 * e + 1], f.y, s0);
                }
              }
              acc[m][b] += s0;
            }
          }
        }
      }
    } else {
      // four chunks of each of the neuron's rows in flight per lane; each
      // widened x chunk serves all of them
      constexpr int U = 4;
      const int nch = p.len / 8;
      const uint8_t* rows[NUP];
#pragma unroll
      for (int m = 0; m < NUP; ++m) rows[m] = (m == 0 ? p.w : p.w2nd) + (size_t)nid * rb;
      for (int c0 = lane; c0 < nch; c0 += 32 * U) {
        uint4 wq[NUP][U];
#pragma unroll
        for (int m = 0; m < NUP; ++m)
#pragma unroll
          for (int u = 0; u < U; ++u) {
            const int c = c0 + 32 * u;
            wq[m][u] = c < nch ? ldg_stream(rows[m] + (size_t)c * 16) : make_uint4(0, 0, 0, 0);
          }
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int c = c0 + 32 * u;
          if (c < nch) {
#pragma unroll
            for (int b = 0; b < BB; ++b) {
              if (b < B) {
                float xf[8];
                if constexpr (MODE == kModePred2) {
                  const float4* ap = reinterpret_cast<const float4*>(p.x32 + (size_t)b * p.len + c * 8);
                  const float4 a0 = __ldg(ap), a1 = __ldg(ap + 1);
                  xf[0] = a0.x; xf[1] = a0.y; xf[2] = a0.z; xf[3] = a0.w;
                  xf[4] = a1.x; xf[5] = a1.y; xf[6] = a1.z; xf[7] = a1.w;
                } else {
                  const uint4 xv = __ldg(reinterpret_cast<const uint4*>(p.x16 + (size_t)b * p.len + c * 8));
                  widen8<XDT>(xv, xf);
                }
#pragma unroll
                for (int m = 0; m < NUP; ++m) acc[m][b] += dot8<WDT == 2 ? 0 : WDT>(wq[m][u], xf);
              }
            }
          }
        }
      }
    }
    // reduce across the warp, 32 tokens at a time
#pragma unroll
    for (int g = 0; g < (BB + 31) / 32; ++g) {
      constexpr int VG = BB < 32 ? BB : 32;
      constexpr int SH = 5 - log2c<VG>();
      float tot[NUP];
#pragma unroll
      for (int m = 0; m < NUP; ++m) {
        float v[VG];
#pragma unroll
        for (int t = 0; t < VG; ++t) v[t] = acc[m][g * 32 + t];
        tot[m] = warp_reduce_transposed<VG>(v);
      }
      const int b = g * 32 + (lane >> SH);
      if ((lane & ((1 << SH) - 1)) == 0 && b < B) {
        const float bias = p.bias ? p.bias[nid] : 0.f;
        if constexpr (MODE == kModePred1) {
          p.out[(size_t)b * p.nrows + row] = fmaxf(tot[0] + bias, 0.f);
        } else if constexpr (MODE == kModePred2) {
          const float s = tot[0] + bias;
          if (p.out) p.out[(size_t)b * p.nrows + row] = s;
          if (s > p.threshold) atomicOr(&p.mask[(size_t)b * (p.nrows / 32) + row / 32], 1u << (row & 31));
        } else {
          float h = fmaxf(tot[0] + (valid ? bias : 0.f), 0.f);
          if constexpr (ACT == 1) h *= tot[NUP - 1];
          if constexpr (ACT == 2) h *= h;
          if (!valid) h = 0.f;
          p.out[(size_t)row * B + b] = h;
        }
      }
    }
  }
}

// ------------------------------------ predictor layer 2, batches of 3 to 15
// One CTA per mask word: rows 32w .. 32w + 31 of W2 (one contiguous slab,
// asked of the L2 before the dependency wait) for 8 tokens of the batch
// (blockIdx.y selects the 8).  The rank is split over NQ warp groups so that
// each lane holds its slice of a for the 8 tokens in registers (64 floats)
// and streams one 16-byte chunk of each row; the NQ partial dots of a row
// meet in shared memory and are added in a fixed order.  Each warp of the
// combine step holds one token and the 32 rows of the word, so one ballot is
// the token's mask word: the mask is written whole, with no atomics.
struct Pred2WordsParams {
  const uint8_t* w2;       // [F x r] 16-bit rows
  const float* b2;         // [F]
  const float* a;          // [B x r] fp32
  uint32_t* mask;          // [B x F/32]
  float* logits;           // [B x F] or null
  float threshold;
  int F, r, B;
};

template <int DT, int NQ, int RU>
__global__ void __launch_bounds__(256) k_pred2_words(Pred2WordsParams p) {
  static_assert(RU == 32 || RU == 16, "a unit is a mask word or half of one");
  constexpr int RS = 8 / NQ;          // row streams
  constexpr int ROWS = RU / RS;       // rows per warp
  constexpr int U = 4;                // rows whose chunks are in flight together
  __shared__ float part[RU][NQ][8];
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  const int q = warp % NQ, rs = warp / NQ;
  const int b0 = blockIdx.y * 8;
  const int nunits = p.F / RU;
  const size_t rb = (size_t)p.r * 2;
  // the CTA takes units blockIdx.x, + gridDim.x, ...: the activations a of
  // its 8 tokens are loaded once and serve every unit (one unit per CTA
  // re-read as many bytes of a from the L2 as of W2)
  auto prefetch_unit = [&](int unit) {  // a unit's rows are contiguous
    const uint8_t* slab = p.w2 + (size_t)unit * RU * rb;
    const size_t bytes = RU * rb;
    for (size_t o = 0; o < bytes; o += 32768)
      prefetch_l2(slab + o, (uint32_t)(bytes - o < 32768 ? bytes - o : 32768));
  };
  if (t == 0 && blockIdx.x < nunits) prefetch_unit(blockIdx.x);
  pdl_wait();
  pdl_trigger();
  const int nch = p.r / 8;
  const int c0 = (int)(((long long)nch * q) / NQ), c1 = (int)(((long long)nch * (q + 1)) / NQ);
  const int c = c0 + lane;
  const bool mine = c < c1;  // at most 32 chunks per group (rank <= 2048)
  float av[8][8];
#pragma unroll
  for (int b = 0; b < 8; ++b) {
    const bool ok = mine && b0 + b < p.B;
    const float4* ap = reinterpret_cast<const float4*>(p.a + (size_t)(b0 + b) * p.r + (size_t)c * 8);
    const float4 lo = ok ? __ldg(ap) : make_float4(0.f, 0.f, 0.f, 0.f);
    const float4 hi = ok ? __ldg(ap + 1) : make_float4(0.f, 0.f, 0.f, 0.f);
    av[b][0] = lo.x; av[b][1] = lo.y; av[b][2] = lo.z; av[b][3] = lo.w;
    av[b][4] = hi.x; av[b][5] = hi.y; av[b][6] = hi.z; av[b][7] = hi.w;
  }
  for (int unit = blockIdx.x; unit < nunits; unit += gridDim.x) {
    if (t == 0 && unit + (int)gridDim.x < nunits) prefetch_unit(unit + gridDim.x);
    const uint8_t* slab = p.w2 + (size_t)unit * RU * rb;
    for (int r0 = 0; r0 < ROWS; r0 += U) {
      uint4 w[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int row = rs * ROWS + r0 + u;
        w[u] = mine ? ldg_stream(slab + (size_t)row * rb + (size_t)c * 16) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        float v[8];
        const uint32_t wv[4] = {w[u].x, w[u].y, w[u].z, w[u].w};
#pragma unroll
        for (int b = 0; b < 8; ++b) {
          float z = 0.f;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = unpack2<DT>(wv[e]);
            z = fmaf(f.x, av[b][2 * e], z);
            z = fmaf(f.y, av[b][2 * e + 1], z);
          }
          v[b] = z;
        }
        const float tot = warp_reduce_transposed<8>(v);  // lane holds token lane / 4
        if ((lane & 3) == 0) part[rs * ROWS + r0 + u][q][lane >> 2] = tot;
      }
    }
    __syncthreads();
    // warp b: token b0 + b, lane = row of the unit.  A half-word unit (RU 16)
    // writes its 16 bits as one half of the little-endian mask word, so two
    // units fill a word without atomics.
    const int b = warp, n = unit * RU + lane;
    if (b0 + b < p.B) {  // warp-uniform
      float sv = 0.f;
      if (lane < RU) {
#pragma unroll
        for (int g = 0; g < NQ; ++g) sv += part[lane][g][b];
        sv += p.b2[n];
        if (p.logits) p.logits[(size_t)(b0 + b) * p.F + n] = sv;
      }
      const uint32_t bits = __ballot_sync(0xffffffffu, lane < RU && sv > p.threshold);
      if (lane == 0) {
        if constexpr (RU == 32)
          p.mask[(size_t)(b0 + b) * (p.F / 32) + unit] = bits;
        else
          reinterpret_cast<uint16_t*>(p.mask)[(size_t)(b0 + b) * (p.F / 16) + unit] =
              (uint16_t)bits;
      }
    }
    __syncthreads();  // part is rewritten by the next unit
  }
}

// ---------------------------------------------------- batched gathered down
// Grid (column slices, neuron slices).  Thread: 8 consecutive columns.  For
// each group of 8 tokens, sums h[k][b] * W_down^T[idx[k]][cols] over the
// neuron slice and writes part[slice][b][cols].
struct DownParams {
  const uint8_t* w_dn;
  const int32_t* idx;
  const int32_t* count;
  const float* h;          // [K x B]
  float* part;             // [gridDim.y x B x d]
  int d, F, B;
  int b0;                  // k_down2: first token of this pass (B is the row stride of h)
};

template <int WDT>
__global__ void __launch_bounds__(256) k_down(DownParams p) {
  pdl_wait();
  pdl_trigger();
  int K = *p.count;
  K = K < 0 ? 0 : (K > p.F ? p.F : K);
  const int S = gridDim.y;
  const int k0 = (int)(((long long)K * blockIdx.y) / S);
  const int k1 = (int)(((long long)K * (blockIdx.y + 1)) / S);
  const int c8 = blockIdx.x * 256 + threadIdx.x;  // unit of 8 columns
  if (c8 >= p.d / 8) return;
  const size_t rb = WDT == 2 ? (size_t)p.d / 32 * 18 : (size_t)p.d * 2;
  for (int b0 = 0; b0 < p.B; b0 += 8) {
    float acc[8][8];
#pragma unroll
    for (int b = 0; b < 8; ++b)
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[b][e] = 0.f;
    for (int k = k0; k < k1; ++k) {
      int nid = p.idx[k];
      if (nid < 0 || nid >= p.F) nid = 0;  // its h is zero (flagged by k_rows)
      const uint8_t* row = p.w_dn + (size_t)nid * rb;
      float wv[8];
      if constexpr (WDT == 2) {
        const int blk = c8 >> 2, sub = c8 & 3;
        const uint16_t* h16 = reinterpret_cast<const uint16_t*>(row + (size_t)blk * 18);
        const float sc = __half2float(__ushort_as_half(h16[0]));
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const uint32_t two = h16[1 + (sub & 1) * 4 + e];
#pragma unroll
          for (int k2 = 0; k2 < 2; ++k2) {
            const uint32_t byte = (two >> (8 * k2)) & 0xffu;
            wv[2 * e + k2] = q4_val(sub < 2 ? (byte & 15u) : (byte >> 4)) * sc;
          }
        }
      } else {
        const uint4 w = __ldg(reinterpret_cast<const uint4*>(row + (size_t)c8 * 16));
        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = unpack2<WDT>(ww[e]);
          wv[2 * e] = f.x;
          wv[2 * e + 1] = f.y;
        }
      }
#pragma unroll
      for (int b = 0; b < 8; ++b) {
        if (b0 + b < p.B) {
          const float hb = __ldg(p.h + (size_t)k * p.B + b0 + b);
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[b][e] = fmaf(hb, wv[e], acc[b][e]);
        }
      }
    }
#pragma unroll
    for (int b = 0; b < 8; ++b) {
      if (b0 + b < p.B) {
        float4* dst = reinterpret_cast<float4*>(p.part + ((size_t)blockIdx.y * p.B + b0 + b) * p.d +
                                                (size_t)c8 * 8);
        dst[0] = make_float4(acc[b][0], acc[b][1], acc[b][2], acc[b][3]);
        dst[1] = make_float4(acc[b][4], acc[b][5], acc[b][6], acc[b][7]);
      }
    }
  }
}

// ------------------------------------- batched gathered down, 16-bit, B % 4 == 0
// One pass over the slice's rows for all tokens: thread t owns CW = 64/BB
// consecutive columns (so BB x CW = 64 fp32 accumulators), four neurons'
// index and row loads are in flight at a time, and the h values of a neuron
// (B floats) are read as float4s that every thread of the CTA shares via L1.
template <int CW>
__device__ __forceinline__ void load_cw(const uint8_t* p, uint32_t (&w)[(CW + 1) / 2]) {
  if constexpr (CW == 8) {
    const uint4 v = ldg_stream(p);
    w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
  } else if constexpr (CW == 4) {
    const uint2 v = __ldg(reinterpret_cast<const uint2*>(p));
    w[0] = v.x; w[1] = v.y;
  } else if constexpr (CW == 2) {
    w[0] = __ldg(reinterpret_cast<const uint32_t*>(p));
  } else {
    w[0] = __ldg(reinterpret_cast<const uint16_t*>(p));
  }
}

template <int WDT, int BB>
__global__ void __launch_bounds__(256) k_down2(DownParams p) {
  constexpr int CW = 64 / BB;          // columns per thread
  constexpr int NW = (CW + 1) / 2;     // 32-bit words per row piece
  constexpr int U = 8;                 // neurons in flight
  pdl_wait();
  pdl_trigger();
  int K = *p.count;
  K = K < 0 ? 0 : (K > p.F ? p.F : K);
  const int S = gridDim.y;
  const int k0 = (int)(((long long)K * blockIdx.y) / S);
  const int k1 = (int)(((long long)K * (blockIdx.y + 1)) / S);
  const int cu = blockIdx.x * blockDim.x + threadIdx.x;  // unit of CW columns
  if (cu * CW >= p.d) return;
  const size_t rb = (size_t)p.d * 2;
  const int B = p.B;
  const int nb = min(BB, B - p.b0);  // tokens of this pass
  float acc[BB][CW];
#pragma unroll
  for (int b = 0; b < BB; ++b)
#pragma unroll
    for (int e = 0; e < CW; ++e) acc[b][e] = 0.f;
  // the next group's neuron ids are requested while this group's rows load
  int nxt[U];
#pragma unroll
  for (int u = 0; u < U; ++u) nxt[u] = k0 + u < k1 ? p.idx[k0 + u] : 0;
  for (int k = k0; k < k1; k += U) {
    int nid[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int v = nxt[u];
      nid[u] = (v < 0 || v >= p.F) ? 0 : v;  // an invalid entry's h is zero
    }
#pragma unroll
    for (int u = 0; u < U; ++u) nxt[u] = k + U + u < k1 ? p.idx[k + U + u] : 0;
    uint32_t w[U][NW];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if (k + u < k1) load_cw<CW>(p.w_dn + (size_t)nid[u] * rb + (size_t)cu * CW * 2, w[u]);
      else
#pragma unroll
        for (int q = 0; q < NW; ++q) w[u][q] = 0u;
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if (k + u < k1) {
        float wf[CW];
        if constexpr (CW == 1) {
          wf[0] = WDT == 0 ? __half2float(__ushort_as_half((unsigned short)w[u][0]))
                           : __uint_as_float(w[u][0] << 16);
        } else {
#pragma unroll
          for (int q = 0; q < NW; ++q) {
            const float2 f = unpack2<WDT>(w[u][q]);
            wf[2 * q] = f.x;
            wf[2 * q + 1] = f.y;
          }
        }
        const float4* hp = reinterpret_cast<const float4*>(p.h + (size_t)(k + u) * B + p.b0);
#pragma unroll
        for (int b4 = 0; b4 < BB / 4; ++b4) {
          if (4 * b4 < nb) {
            const float4 hv = __ldg(hp + b4);
            const float hb[4] = {hv.x, hv.y, hv.z, hv.w};
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
              for (int e = 0; e < CW; ++e) acc[4 * b4 + i][e] = fmaf(hb[i], wf[e], acc[4 * b4 + i][e]);
          }
        }
      }
    }
  }
#pragma unroll
  for (int b = 0; b < BB; ++b) {
    if (b < nb) {
      float* dst = p.part + ((size_t)blockIdx.y * B + p.b0 + b) * p.d + (size_t)cu * CW;
#pragma unroll
      for (int e = 0; e < CW; ++e) dst[e] = acc[b][e];
    }
  }
}

// --------------------------------- batched row GEMM on tensor cores (mma.sync)
// For batches of 8 or more tokens, the rows-times-activations products of the
// predictor's first layer and of the gathered up projection are small GEMMs:
// D[16 neurons x 8 tokens] += A[16 x 16] B[16 x 8] with m16n8k16 (fp32
// accumulate, so products of 16-bit values are exact).  A warp takes a tile
// of 16 rows and walks the row length in steps of 32 elements.  The
// contraction index is permuted the same way in A and B so that each lane's
// A fragment is 16 contiguous bytes of one row and its B fragment 16
// contiguous bytes of one token: lane (g = lane/4, t = lane%4) loads
// elements [32s + 8t, 32s + 8t + 8) of rows g and g+8 (words W0..W3) and of
// token g of each 8-token tile (words X0..X3); k-step 2s uses (W0, W1 | X0,
// X1), k-step 2s+1 uses (W2, W3 | X2, X3).  Over t = 0..3 the four word
// slots cover the 32 elements of the step exactly once.
template <int WDT>
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  if constexpr (WDT == 0)
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  else
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// MODE kModePred1: rows = W1 (dense), out a[b x r] = relu(. + b1).
// MODE kModeUp:    rows = idx-gathered activation rows (and W_up for ReGLU),
//                  out h[k x B].  NT = 8-token tiles (B <= 8 NT).
// One CTA per tile of 16 rows; its 8 warps split the row length (warp w takes
// steps [w S/8, (w+1) S/8)), and the 8 partial accumulators are added in warp
// order through shared memory, so the sum is reproducible.
constexpr int kMmaWarps = 8;

template <int MODE, int WDT, int ACT, int NT>
__global__ void __launch_bounds__(32 * kMmaWarps) k_rows_mma(RowsParams p) {
  static_assert(WDT == 0 || WDT == 1, "16-bit rows");
  constexpr int NUP = (MODE == kModeUp && ACT == 1) ? 2 : 1;
  constexpr int NV = NUP * NT * 4;  // accumulator values per lane
  constexpr int U = 4;              // 32-element steps whose loads are in flight together
  extern __shared__ __align__(16) float part_s[];  // [kMmaWarps][NV][32]
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, g = lane >> 2, t = lane & 3;
  int nrows = p.nrows;
  if (MODE == kModeUp) {
    const int K = *p.count;
    nrows = K < 0 ? 0 : (K > p.nrows ? p.nrows : K);
  }
  const int tile = blockIdx.x;
  if (tile * 16 >= nrows) return;  // whole CTA: no barrier is skipped by part of it
  const int B = p.B;
  const int len = p.len;
  // the contraction in 32-element steps: slice blockIdx.y of gridDim.y (the
  // predictor's layer 1 has only r/16 tiles), then split among the warps
  const int nsteps = len / 32;
  const int Y = gridDim.y;
  const int c_lo = (int)(((long long)nsteps * blockIdx.y) / Y);
  const int c_n = (int)(((long long)nsteps * (blockIdx.y + 1)) / Y) - c_lo;
  const int s_lo = c_lo + (int)(((long long)c_n * warp) / kMmaWarps);
  const int s_hi = c_lo + (int)(((long long)c_n * (warp + 1)) / kMmaWarps);
  const size_t rb = (size_t)len * 2;
  const uint64_t pol = policy_evict_first();

  int nid[2];
  bool ok[2];
#pragma unroll
  for (int hlf = 0; hlf < 2; ++hlf) {
    const int row = tile * 16 + g + 8 * hlf;
    int v = row;
    bool valid = row < nrows;
    if (MODE == kModeUp && valid) {
      v = p.idx[row];
      if (v < 0 || v >= p.nrows) {
        if (warp == 0) set_error(kErrBadIndex);
        valid = false;
      }
    }
    nid[hlf] = valid ? v : 0;
    ok[hlf] = valid;
  }
  float acc[NUP][NT][4];
#pragma unroll
  for (int m = 0; m < NUP; ++m)
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[m][n][e] = 0.f;

  for (int s0 = s_lo; s0 < s_hi; s0 += U) {
    uint4 wa[NUP][U][2];
#pragma unroll
    for (int m = 0; m < NUP; ++m)
#pragma unroll
      for (int u = 0; u < U; ++u)
#pragma unroll
        for (int hlf = 0; hlf < 2; ++hlf) {
          const int s = s0 + u;
          const uint8_t* row = (m == 0 ? p.w : p.w2nd) + (size_t)nid[hlf] * rb;
          wa[m][u][hlf] = (s < s_hi && ok[hlf])
                              ? ldg_stream_hint(row + (size_t)s * 64 + (size_t)t * 16, pol)
                              : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int s = s0 + u;
      if (s < s_hi) {
#pragma unroll
        for (int n = 0; n < NT; ++n) {
          const int tok = n * 8 + g;
          const uint4 xv = tok < B ? __ldg(reinterpret_cast<const uint4*>(
                                         p.x16 + (size_t)tok * len + (size_t)s * 32 + t * 8))
                                   : make_uint4(0, 0, 0, 0);
#pragma unroll
          for (int m = 0; m < NUP; ++m) {
            const uint32_t a0[4] = {wa[m][u][0].x, wa[m][u][1].x, wa[m][u][0].y, wa[m][u][1].y};
            const uint32_t a1[4] = {wa[m][u][0].z, wa[m][u][1].z, wa[m][u][0].w, wa[m][u][1].w};
            mma16816<WDT>(acc[m][n], a0, xv.x, xv.y);
            mma16816<WDT>(acc[m][n], a1, xv.z, xv.w);
          }
        }
      }
    }
  }

  // the warps' partial sums, added in warp order
#pragma unroll
  for (int m = 0; m < NUP; ++m)
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) part_s[((size_t)warp * NV + (m * NT + n) * 4 + e) * 32 + lane] = acc[m][n][e];
  __syncthreads();
  if (warp != 0) return;
#pragma unroll
  for (int m = 0; m < NUP; ++m)
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float v = 0.f;
#pragma unroll
        for (int w = 0; w < kMmaWarps; ++w) v += part_s[((size_t)w * NV + (m * NT + n) * 4 + e) * 32 + lane];
        acc[m][n][e] = v;
      }

  // epilogue: c0,c1 -> row g, tokens 2t, 2t+1; c2,c3 -> row g+8
#pragma unroll
  for (int n = 0; n < NT; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int hlf = e >> 1;
      const int row = tile * 16 + g + 8 * hlf;
      const int tok = n * 8 + 2 * t + (e & 1);
      if (row < nrows && tok < B) {
        const float bias = p.bias ? p.bias[nid[hlf]] : 0.f;
        if (MODE == kModePred1 && Y > 1) {
          p.part[((size_t)blockIdx.y * B + tok) * p.nrows + row] = acc[0][n][e];
        } else if constexpr (MODE == kModePred1) {
          const float a = fmaxf(acc[0][n][e] + bias, 0.f);
          p.out[(size_t)tok * p.nrows + row] = a;
        } else {
          float h = fmaxf(acc[0][n][e] + (ok[hlf] ? bias : 0.f), 0.f);
          if constexpr (ACT == 1) h *= acc[NUP - 1][n][e];
          if constexpr (ACT == 2) h *= h;
          if (!ok[hlf]) h = 0.f;
          p.out[(size_t)row * B + tok] = h;
        }
      }
    }
}

}  // namespace pi
