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

#pragma unroll
    for (int m = 0; m < NUP; ++m) {
      const uint8_t* rowp = (m == 0 ? p.w : p.w2nd) + (size_t)nid * rb;
      if constexpr (WDT == 2) {
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
      } else {
        for (int c = lane; c < p.len / 8; c += 32) {
          const uint4 w = __ldg(reinterpret_cast<const uint4*>(rowp + (size_t)c * 16));
#pragma unroll
          for (int b = 0; b < BB; ++b) {
            if (b < B) {
              if constexpr (MODE == kModePred2) {
                const float4* ap = reinterpret_cast<const float4*>(p.x32 + (size_t)b * p.len + c * 8);
                const float4 a0 = __ldg(ap), a1 = __ldg(ap + 1);
                const float2 f0 = unpack2<WDT>(w.x), f1 = unpack2<WDT>(w.y);
                const float2 f2 = unpack2<WDT>(w.z), f3 = unpack2<WDT>(w.w);
                float s = acc[m][b];
                s = fmaf(f0.x, a0.x, s); s = fmaf(f0.y, a0.y, s);
                s = fmaf(f1.x, a0.z, s); s = fmaf(f1.y, a0.w, s);
                s = fmaf(f2.x, a1.x, s); s = fmaf(f2.y, a1.y, s);
                s = fmaf(f3.x, a1.z, s); s = fmaf(f3.y, a1.w, s);
                acc[m][b] = s;
              } else {
                const uint4 xv = __ldg(reinterpret_cast<const uint4*>(p.x16 + (size_t)b * p.len + c * 8));
                float xf[8];
                widen8<XDT>(xv, xf);
                acc[m][b] += dot8<WDT == 2 ? 0 : WDT>(w, xf);
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

}  // namespace pi
