// Compaction and the gathered (neuron-aware) FFN.
//
// PowerInfer keeps, per layer, a table that maps each active neuron to its
// original row (unite.ai page, "Neuronen-Platzierung und -Verwaltung"), and
// its neuron-aware operator computes only those neurons' row vectors of W_up
// (and W_gate) and W_down^T, with no sparse-format conversion (same page,
// "Neuronenbewusster Operator").  Here W_down is stored transposed, so a
// neuron's down-projection column is one contiguous row too, and every
// gathered read is a single contiguous bulk copy.
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

// ------------------------------------------------------ gathered FFN, fused
// Each CTA takes a contiguous, balanced slice [k0, k1) of the K listed
// neurons.  A stage holds one neuron: its activation row (W_up for ReLU,
// W_gate for ReGLU), its W_up row (ReGLU only) and its W_down^T row.  The
// consumers compute h for a group of kGroup neurons (block-wide dot products),
// then add h * W_down^T[n] into fp32 accumulators that stay in registers for
// the whole slice.  The CTA's partial y goes to part[cta]; a fixed-order
// reduction (k_reduce) sums the partials, so there are no atomics and the
// result is bit-reproducible.
constexpr int kGroup = 4;

struct FfnParams {
  const uint8_t* w_act;    // W_up (ReLU) or W_gate (ReGLU)
  const uint8_t* w_up;     // W_up (ReGLU only)
  const uint8_t* w_dn;     // W_down^T
  const float* b_act;      // b_up (ReLU) / b_gate (ReGLU), or null
  const uint16_t* x;       // [B x d]
  const int32_t* idx;
  const int32_t* count;
  float* part;             // [gridDim.x x B x d]
  int d, F;
  uint32_t row_bytes;
  int nstages;
};

// WDT: 0 fp16, 1 bf16, 2 Q4_0 (with fp16 activations).  ACT: 0 ReLU, 1 ReGLU.
// CPT: units per consumer thread (a unit is 8 elements for 16-bit weights, one
// 32-element block for Q4_0).
template <int WDT, int ACT, int B, int CPT>
__global__ void __launch_bounds__(kThreads, 1) k_ffn(FfnParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr int NM = ACT == 1 ? 3 : 2;      // matrices per stage
  constexpr int NUP = ACT == 1 ? 2 : 1;     // dot products per neuron
  constexpr int V = kGroup * NUP * B;       // values reduced per group
  constexpr int SH = 5 - log2c<V>();
  constexpr int XDT = WDT == 1 ? 1 : 0;     // activation dtype
  constexpr int UE = WDT == 2 ? 32 : 8;     // elements per unit
  const int NS = p.nstages;

  uint64_t* full = reinterpret_cast<uint64_t*>(smem);
  uint64_t* empty = full + NS;
  float* meta_bias = reinterpret_cast<float*>(empty + NS);     // [NS]
  int* meta_ok = reinterpret_cast<int*>(meta_bias + NS);       // [NS]
  float* red = reinterpret_cast<float*>(smem + 1024);          // [2][8][V]
  float* hs = red + 2 * kConsumerWarps * V;                    // [2][kGroup * B]
  uint8_t* stages = smem + 1024 + 2 * kConsumerWarps * V * 4 + 2 * kGroup * B * 4;
  stages = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(stages) + 127) & ~uintptr_t(127));
  const uint32_t rb = p.row_bytes;
  const uint32_t stage_bytes = rb * NM;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumerWarps);
    }
    fence_mbar_init();
  }
  __syncthreads();
  pdl_trigger();
  pdl_wait();  // idx, count and x come from earlier kernels

  int K = *p.count;
  K = K < 0 ? 0 : (K > p.F ? p.F : K);
  const int G = gridDim.x;
  const int k0 = (int)(((long long)K * blockIdx.x) / G);
  const int k1 = (int)(((long long)K * (blockIdx.x + 1)) / G);
  const int n = k1 - k0;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp == 0) {
    // ---------------------------------------------------------- producer
    const uint64_t pol = policy_evict_first();
    bool ok = true;
    for (int base = 0; base < n && ok; base += 32) {
      int nid = 0, valid = 0;
      float bias = 0.f;
      if (base + lane < n) {
        nid = p.idx[k0 + base + lane];
        valid = (nid >= 0 && nid < p.F);
        if (!valid) {
          set_error(kErrBadIndex);
          nid = 0;
        }
        bias = (p.b_act && valid) ? p.b_act[nid] : 0.f;
      }
      const int cnt = min(32, n - base);
      for (int j = 0; j < cnt; ++j) {
        const int nj = __shfl_sync(0xffffffffu, nid, j);
        const int vj = __shfl_sync(0xffffffffu, valid, j);
        const float bj = __shfl_sync(0xffffffffu, bias, j);
        if (lane == 0 && ok) {
          const int i = base + j;
          const int s = i % NS;
          if (i >= NS && !mbar_wait(&empty[s], ((i / NS) - 1) & 1)) {
            ok = false;
          } else {
            meta_bias[s] = bj;
            meta_ok[s] = vj;
            mbar_arrive_expect_tx(&full[s], stage_bytes);
            uint8_t* st = stages + (size_t)s * stage_bytes;
            const size_t off = (size_t)nj * rb;
            bulk_g2s_hint(st, p.w_act + off, rb, &full[s], pol);
            if constexpr (ACT == 1) bulk_g2s_hint(st + rb, p.w_up + off, rb, &full[s], pol);
            bulk_g2s_hint(st + (NM - 1) * rb, p.w_dn + off, rb, &full[s], pol);
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
      }
    }
    if (lane == 0)
      for (int i = max(0, n - NS); i < n; ++i) mbar_wait(&full[i % NS], (i / NS) & 1);
    return;
  }

  // ------------------------------------------------------------ consumers
  const int ct = threadIdx.x - 32;
  const int cw = warp - 1;
  const int nunits = p.d / UE;

  // activations of this thread's units, per token
  constexpr int XW = WDT == 2 ? 32 : 4;  // Q4: 32 fp32 values; 16-bit: 4 packed words
  uint32_t xr[B][CPT][XW];
#pragma unroll
  for (int b = 0; b < B; ++b)
#pragma unroll
    for (int c = 0; c < CPT; ++c) {
      const int u = ct + kConsumers * c;
      if constexpr (WDT == 2) {
#pragma unroll
        for (int e = 0; e < 32; ++e)
          xr[b][c][e] = (u < nunits) ? __float_as_uint(__half2float(__ushort_as_half(
                                           p.x[(size_t)b * p.d + u * 32 + e])))
                                     : 0u;
      } else {
        uint4 v = make_uint4(0, 0, 0, 0);
        if (u < nunits) v = *reinterpret_cast<const uint4*>(p.x + (size_t)b * p.d + u * 8);
        xr[b][c][0] = v.x; xr[b][c][1] = v.y; xr[b][c][2] = v.z; xr[b][c][3] = v.w;
      }
    }

  float acc[B][CPT][UE];
#pragma unroll
  for (int b = 0; b < B; ++b)
#pragma unroll
    for (int c = 0; c < CPT; ++c)
#pragma unroll
      for (int e = 0; e < UE; ++e) acc[b][c][e] = 0.f;

  bool ok = true;
  int grp = 0;
  for (int g = 0; g < n; g += kGroup, ++grp) {
    const int ng = min(kGroup, n - g);
    const int buf = grp & 1;
#pragma unroll
    for (int q = 0; q < kGroup; ++q) {
      const int i = g + q;
      if (q < ng && ok && !mbar_wait(&full[i % NS], (i / NS) & 1)) ok = false;
    }
    // partial dot products of this thread's units
    float v[V];
#pragma unroll
    for (int t = 0; t < V; ++t) v[t] = 0.f;
    if (ok) {
#pragma unroll
      for (int q = 0; q < kGroup; ++q) {
        if (q < ng) {
          const uint8_t* st = stages + (size_t)((g + q) % NS) * stage_bytes;
#pragma unroll
          for (int m = 0; m < NUP; ++m) {
            const uint8_t* row = st + m * rb;
#pragma unroll
            for (int c = 0; c < CPT; ++c) {
              const int u = ct + kConsumers * c;
              if (u < nunits) {
                if constexpr (WDT == 2) {
                  const uint8_t* blk = row + (size_t)u * 18;
                  const uint16_t* h16 = reinterpret_cast<const uint16_t*>(blk);
                  const float sc = __half2float(__ushort_as_half(h16[0]));
                  uint32_t qb[4];
#pragma unroll
                  for (int e = 0; e < 4; ++e)
                    qb[e] = (uint32_t)h16[1 + 2 * e] | ((uint32_t)h16[2 + 2 * e] << 16);
#pragma unroll
                  for (int b = 0; b < B; ++b) {
                    float s0 = 0.f, s1 = 0.f;
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                      const uint32_t byte = (qb[e >> 2] >> ((e & 3) * 8)) & 0xffu;
                      s0 = fmaf(q4_val(byte & 15u), __uint_as_float(xr[b][c][e]), s0);
                      s1 = fmaf(q4_val(byte >> 4), __uint_as_float(xr[b][c][e + 16]), s1);
                    }
                    v[(q * NUP + m) * B + b] += (s0 + s1) * sc;
                  }
                } else {
                  const uint4 w = *reinterpret_cast<const uint4*>(row + (size_t)u * 16);
#pragma unroll
                  for (int b = 0; b < B; ++b) {
                    float a0 = 0.f, a1 = 0.f;
                    dot2<XDT>(w.x, xr[b][c][0], a0, a1);
                    dot2<XDT>(w.y, xr[b][c][1], a0, a1);
                    dot2<XDT>(w.z, xr[b][c][2], a0, a1);
                    dot2<XDT>(w.w, xr[b][c][3], a0, a1);
                    v[(q * NUP + m) * B + b] += a0 + a1;
                  }
                }
              }
            }
          }
        }
      }
    }
    // block reduction: warp transposed reduce, then across warps
    const float tot = warp_reduce_transposed<V>(v);
    if ((lane & ((1 << SH) - 1)) == 0) red[(buf * kConsumerWarps + cw) * V + (lane >> SH)] = tot;
    named_bar_sync(1, kConsumers);
    if (ct < kGroup * B) {
      const int q = ct / B, b = ct % B;
      float h = 0.f;
      if (q < ng && ok) {
        float sa = 0.f, su = 0.f;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) {
          sa += red[(buf * kConsumerWarps + w) * V + (q * NUP + 0) * B + b];
          if constexpr (ACT == 1) su += red[(buf * kConsumerWarps + w) * V + (q * NUP + 1) * B + b];
        }
        const int s = (g + q) % NS;
        const float pre = sa + meta_bias[s];
        h = fmaxf(pre, 0.f);
        if constexpr (ACT == 1) h *= su;
        if (!meta_ok[s]) h = 0.f;
      }
      hs[buf * kGroup * B + ct] = h;
    }
    named_bar_sync(1, kConsumers);
    // down projection: acc += h * W_down^T[n]
    if (ok) {
#pragma unroll
      for (int q = 0; q < kGroup; ++q) {
        if (q < ng) {
          const uint8_t* row = stages + (size_t)((g + q) % NS) * stage_bytes + (NM - 1) * rb;
          float hq[B];
#pragma unroll
          for (int b = 0; b < B; ++b) hq[b] = hs[buf * kGroup * B + q * B + b];
#pragma unroll
          for (int c = 0; c < CPT; ++c) {
            const int u = ct + kConsumers * c;
            if (u < nunits) {
              if constexpr (WDT == 2) {
                const uint8_t* blk = row + (size_t)u * 18;
                const uint16_t* h16 = reinterpret_cast<const uint16_t*>(blk);
                const float sc = __half2float(__ushort_as_half(h16[0]));
                uint32_t qb[4];
#pragma unroll
                for (int e = 0; e < 4; ++e)
                  qb[e] = (uint32_t)h16[1 + 2 * e] | ((uint32_t)h16[2 + 2 * e] << 16);
#pragma unroll
                for (int b = 0; b < B; ++b) {
                  const float hsc = hq[b] * sc;
#pragma unroll
                  for (int e = 0; e < 16; ++e) {
                    const uint32_t byte = (qb[e >> 2] >> ((e & 3) * 8)) & 0xffu;
                    acc[b][c][e] = fmaf(hsc, q4_val(byte & 15u), acc[b][c][e]);
                    acc[b][c][e + 16] = fmaf(hsc, q4_val(byte >> 4), acc[b][c][e + 16]);
                  }
                }
              } else {
                const uint4 w = *reinterpret_cast<const uint4*>(row + (size_t)u * 16);
                const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  const float2 f = unpack2<WDT>(wv[e]);
#pragma unroll
                  for (int b = 0; b < B; ++b) {
                    acc[b][c][2 * e] = fmaf(hq[b], f.x, acc[b][c][2 * e]);
                    acc[b][c][2 * e + 1] = fmaf(hq[b], f.y, acc[b][c][2 * e + 1]);
                  }
                }
              }
            }
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0)
      for (int q = 0; q < ng; ++q) mbar_arrive(&empty[(g + q) % NS]);
  }

  // partial y of this CTA
#pragma unroll
  for (int b = 0; b < B; ++b)
#pragma unroll
    for (int c = 0; c < CPT; ++c) {
      const int u = ct + kConsumers * c;
      if (u < nunits) {
        float4* dst = reinterpret_cast<float4*>(p.part + ((size_t)blockIdx.x * B + b) * p.d +
                                                (size_t)u * UE);
#pragma unroll
        for (int e = 0; e < UE / 4; ++e)
          dst[e] = make_float4(acc[b][c][4 * e], acc[b][c][4 * e + 1], acc[b][c][4 * e + 2],
                               acc[b][c][4 * e + 3]);
      }
    }
}

// ------------------------------------------------------ partial reduction
// out[i] = sum over g = 0..G-1 (in this order within each of 8 slices, the
// slices then added in order) of part[g][i]; MODE 0 writes y, MODE 1 adds into
// the residual stream.  n4 = number of float4 columns (B*d/4).
template <int MODE>
__global__ void __launch_bounds__(256) k_reduce(const float* __restrict__ part, int G, int n4,
                                                float* __restrict__ out) {
  __shared__ float4 sm[8][32];
  pdl_wait();
  pdl_trigger();
  const int col = blockIdx.x * 32 + (threadIdx.x & 31);
  const int sl = threadIdx.x >> 5;
  float4 t = make_float4(0.f, 0.f, 0.f, 0.f);
  if (col < n4) {
    const float4* src = reinterpret_cast<const float4*>(part);
    for (int g = sl; g < G; g += 8) {
      const float4 v = src[(size_t)g * n4 + col];
      t.x += v.x; t.y += v.y; t.z += v.z; t.w += v.w;
    }
  }
  sm[sl][threadIdx.x & 31] = t;
  __syncthreads();
  if (sl == 0 && col < n4) {
    float4 r = sm[0][threadIdx.x];
#pragma unroll
    for (int k = 1; k < 8; ++k) {
      const float4 v = sm[k][threadIdx.x];
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

}  // namespace pi
