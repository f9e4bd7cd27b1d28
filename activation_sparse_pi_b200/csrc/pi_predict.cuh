// Predictor kernels: a = relu(W1 x + b1), s = W2 a + b2, mask = s > threshold.
//
// PowerInfer's online predictor scores every FFN neuron per token and layer
// so that only neurons predicted active are computed (unite.ai page,
// "Adaptive Sparsity-Prädiktoren"; machine-heart page, Figure 8).
//
// Both layers are GEMVs over static weights.  One producer warp streams the
// weight rows into a ring of shared-memory stages with 1-D bulk copies; it
// needs nothing from the previous kernel, so under programmatic dependent
// launch the weights are already arriving while that kernel finishes.  The
// eight consumer warps wait for the previous kernel (griddepcontrol.wait)
// only before they read the activations.
#pragma once
#include "pi_common.cuh"

namespace pi {

constexpr int kConsumerWarps = 8;
constexpr int kConsumers = kConsumerWarps * 32;
constexpr int kThreads = kConsumers + 32;  // + one producer warp
constexpr float kRmsEps = 1e-6f;

// ------------------------------------------------------------------ layer 1
struct Pred1Params {
  const uint8_t* w1;       // [r x d] 16-bit rows
  const float* b1;         // [r] or null
  const uint16_t* x;       // [B x d] 16-bit input (when x_resid is null)
  const float* x_resid;    // [B x d] fp32 residual stream, or null
  uint16_t* x_out;         // [B x d] rounded layer input (written when x_resid)
  float* a;                // [B x r]
  int d, r;
  int rows_per_cta;
  int nstages;
};

// Layer input from the residual stream: x_l = round16(x / sqrt(mean(x^2) +
// eps)) per token.  Every CTA computes it the same way (fixed summation
// order), so all CTAs hold identical x_l.  The residual is read once, with
// 16-byte loads, and kept in registers between the reduction and the cast.
template <int DT, int B>
__device__ void rms_cast_to_smem(const float* __restrict__ xr, uint16_t* xs, int d,
                                 float* red /* >= [kConsumerWarps * B] */, uint16_t* x_out) {
  // float4 per thread: d <= 8192 at B <= 2; the fused predictor takes B = 4 only for d <= 4096
  constexpr int MAXV = (B == 4 ? 4096 : 8192) / (4 * kConsumers);
  const int ct = threadIdx.x - 32;
  const int lane = threadIdx.x & 31, w = ct >> 5;
  const int n4 = d / 4;
  float4 v[B][MAXV];
  float ss[B];
#pragma unroll
  for (int b = 0; b < B; ++b) {
#pragma unroll
    for (int k = 0; k < MAXV; ++k) {
      const int j = ct + kConsumers * k;
      v[b][k] = j < n4 ? reinterpret_cast<const float4*>(xr + (size_t)b * d)[j]
                       : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    float t = 0.f;
#pragma unroll
    for (int k = 0; k < MAXV; ++k) {
      t = fmaf(v[b][k].x, v[b][k].x, t);
      t = fmaf(v[b][k].y, v[b][k].y, t);
      t = fmaf(v[b][k].z, v[b][k].z, t);
      t = fmaf(v[b][k].w, v[b][k].w, t);
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
    ss[b] = t;
  }
  if (lane == 0)
#pragma unroll
    for (int b = 0; b < B; ++b) red[w * B + b] = ss[b];
  named_bar_sync(1, kConsumers);
#pragma unroll
  for (int b = 0; b < B; ++b) {
    float t = 0.f;
#pragma unroll
    for (int i = 0; i < kConsumerWarps; ++i) t += red[i * B + b];
    const float rms = sqrtf(t / (float)d + kRmsEps);
#pragma unroll
    for (int k = 0; k < MAXV; ++k) {
      const int j = ct + kConsumers * k;
      if (j < n4) {
        const uint32_t lo = (uint32_t)round16<DT>(v[b][k].x / rms) |
                            ((uint32_t)round16<DT>(v[b][k].y / rms) << 16);
        const uint32_t hi = (uint32_t)round16<DT>(v[b][k].z / rms) |
                            ((uint32_t)round16<DT>(v[b][k].w / rms) << 16);
        const uint2 pk = make_uint2(lo, hi);
        reinterpret_cast<uint2*>(xs + (size_t)b * d)[j] = pk;
        if (x_out) reinterpret_cast<uint2*>(x_out + (size_t)b * d)[j] = pk;
      }
    }
  }
}

// All eight consumer warps work on every row (x stays in registers, one block
// reduction per group of kRowGroup rows), so the stage ring is consumed in
// order and no warp ever waits on a stage phase ahead of the others.
constexpr int kRowGroup = 4;

template <int DT, int B, int CPT>
__global__ void __launch_bounds__(kThreads, 1) k_pred1(Pred1Params p) {
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr int V = kRowGroup * B;
  constexpr int SH = 5 - log2c<V>();
  const int NS = p.nstages;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem);
  uint64_t* empty = full + NS;
  float* red = reinterpret_cast<float*>(empty + NS);  // [2][8][V] (also rms scratch)
  uint16_t* xs = reinterpret_cast<uint16_t*>(smem + 2048);
  const size_t xbytes = ((size_t)B * p.d * 2 + 127) & ~size_t(127);
  uint8_t* stages = smem + 2048 + xbytes;
  const uint32_t row_bytes = (uint32_t)p.d * 2;

  const int j0 = blockIdx.x * p.rows_per_cta;
  const int j1 = min(p.r, j0 + p.rows_per_cta);
  const int n = max(0, j1 - j0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumerWarps);
    }
    fence_mbar_init();
  }
  __syncthreads();
  pdl_trigger();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp == 0) {
    // producer: weights only, no dependency on the previous kernel
    if (lane == 0) {
      for (int i = 0; i < n; ++i) {
        const int s = i % NS;
        if (i >= NS && !mbar_wait_sleep(&empty[s], ((i / NS) - 1) & 1)) break;
        mbar_arrive_expect_tx(&full[s], row_bytes);
        bulk_g2s(stages + (size_t)s * row_bytes, p.w1 + (size_t)(j0 + i) * row_bytes, row_bytes,
                 &full[s]);
      }
      // drain: no copy may still be in flight when the CTA exits
      for (int i = max(0, n - NS); i < n; ++i) mbar_wait_sleep(&full[i % NS], (i / NS) & 1);
    }
    return;
  }

  // consumers
  pdl_wait();
  const int ct = threadIdx.x - 32;
  const int cw = warp - 1;
  if (p.x_resid) {
    rms_cast_to_smem<DT, B>(p.x_resid, xs, p.d, red, blockIdx.x == 0 ? p.x_out : nullptr);
  } else {
    const uint4* src = reinterpret_cast<const uint4*>(p.x);
    uint4* dst = reinterpret_cast<uint4*>(xs);
    for (int c = ct; c < B * p.d / 8; c += kConsumers) dst[c] = src[c];
  }
  named_bar_sync(1, kConsumers);

  const int nchunks = p.d / 8;
  float xr[B][CPT][8];  // this thread's activations, widened once to fp32
#pragma unroll
  for (int b = 0; b < B; ++b)
#pragma unroll
    for (int c = 0; c < CPT; ++c) {
      const int u = ct + kConsumers * c;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (u < nchunks) v = *reinterpret_cast<const uint4*>(xs + (size_t)b * p.d + u * 8);
      widen8<DT>(v, xr[b][c]);
    }

  bool ok = true;
  int grp = 0;
  for (int g = 0; g < n; g += kRowGroup, ++grp) {
    const int ng = min(kRowGroup, n - g);
    const int buf = grp & 1;
#pragma unroll
    for (int q = 0; q < kRowGroup; ++q) {
      const int i = g + q;
      if (q < ng && ok && !mbar_wait_sleep(&full[i % NS], (i / NS) & 1)) ok = false;
    }
    float v[V];
#pragma unroll
    for (int t = 0; t < V; ++t) v[t] = 0.f;
    if (ok) {
#pragma unroll
      for (int q = 0; q < kRowGroup; ++q) {
        if (q < ng) {
          const uint8_t* row = stages + (size_t)((g + q) % NS) * row_bytes;
#pragma unroll
          for (int c = 0; c < CPT; ++c) {
            const int u = ct + kConsumers * c;
            if (u < nchunks) {
              const uint4 w = *reinterpret_cast<const uint4*>(row + (size_t)u * 16);
#pragma unroll
              for (int b = 0; b < B; ++b) v[q * B + b] += dot8<DT>(w, xr[b][c]);
            }
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0)
      for (int q = 0; q < ng; ++q) mbar_arrive(&empty[(g + q) % NS]);
    const float tot = warp_reduce_transposed<V>(v);
    if ((lane & ((1 << SH) - 1)) == 0) red[(buf * kConsumerWarps + cw) * V + (lane >> SH)] = tot;
    named_bar_sync(1, kConsumers);
    if (ct < V && ok) {
      const int q = ct / B, b = ct % B;
      if (q < ng) {
        float z = 0.f;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) z += red[(buf * kConsumerWarps + w) * V + ct];
        const int j = j0 + g + q;
        z += p.b1 ? p.b1[j] : 0.f;
        p.a[(size_t)b * p.r + j] = fmaxf(z, 0.f);
      }
    }
  }
}

// ------------------------------------------------------------------ layer 2
// Rows are processed in units of 32 (one mask word per token).  A stage holds
// 8 rows; warp w handles rows 4w..4w+3 of each unit.
struct Pred2Params {
  const uint8_t* w2;       // [F x r] 16-bit rows
  const float* b2;         // [F]
  const float* a;          // [B x r] fp32
  uint32_t* mask;          // [B x F/32]
  float* logits;           // [B x F] or null
  float threshold;
  int F, r;
  int units_per_cta;       // units of 32 rows
  int nstages;             // stages of 8 rows
};

template <int DT, int B, int CPL>
__global__ void __launch_bounds__(kThreads, 1) k_pred2(Pred2Params p) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int NS = p.nstages;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem);
  uint64_t* empty = full + NS;
  uint32_t* words = reinterpret_cast<uint32_t*>(empty + NS);  // [2][B]
  float* bias = reinterpret_cast<float*>(smem + 1024);          // [units_per_cta * 32]
  uint8_t* stages = smem + 1024 + (((size_t)p.units_per_cta * 32 * 4 + 127) & ~size_t(127));
  const uint32_t row_bytes = (uint32_t)p.r * 2;
  const uint32_t stage_bytes = row_bytes * 8;

  const int nunits = p.F / 32;
  const int u0 = blockIdx.x * p.units_per_cta;
  const int u1 = min(nunits, u0 + p.units_per_cta);
  const int nu = max(0, u1 - u0);
  const int nst = nu * 4;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 2);
    }
    fence_mbar_init();
  }
  if (threadIdx.x < 2 * B) words[threadIdx.x] = 0u;
  __syncthreads();
  pdl_trigger();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp == 0) {
    if (lane == 0) {
      const uint8_t* base = p.w2 + (size_t)u0 * 32 * row_bytes;
      // stages beyond the ring: ask the L2 for them now, while the previous
      // kernel still runs, so the refills after the ring drains hit the L2
      for (int i = NS; i < nst; ++i) prefetch_l2(base + (size_t)i * stage_bytes, stage_bytes);
      for (int i = 0; i < nst; ++i) {
        const int s = i % NS;
        if (i >= NS && !mbar_wait_sleep(&empty[s], ((i / NS) - 1) & 1)) break;
        mbar_arrive_expect_tx(&full[s], stage_bytes);
        bulk_g2s(stages + (size_t)s * stage_bytes, base + (size_t)i * stage_bytes, stage_bytes,
                 &full[s]);
      }
      for (int i = max(0, nst - NS); i < nst; ++i) mbar_wait_sleep(&full[i % NS], (i / NS) & 1);
    }
    return;
  }

  const int ct = threadIdx.x - 32;
  const int cw = warp - 1;
  // static bias of this CTA's rows (before the dependency wait)
  for (int t = ct; t < nu * 32; t += kConsumers) bias[t] = p.b2[(size_t)u0 * 32 + t];

  pdl_wait();
  // this lane's slice of a: chunks c = lane + 32 k, 8 values each
  const int nch = p.r / 8;
  float av[B][CPL][8];
#pragma unroll
  for (int b = 0; b < B; ++b)
#pragma unroll
    for (int k = 0; k < CPL; ++k) {
      const int c = lane + 32 * k;
#pragma unroll
      for (int e = 0; e < 8; ++e)
        av[b][k][e] = (c < nch) ? p.a[(size_t)b * p.r + c * 8 + e] : 0.f;
    }
  named_bar_sync(1, kConsumers);  // bias visible

  constexpr int V = 4 * B;
  constexpr int SH = 5 - log2c<V>();
  // Every consumer takes part in every unit's barrier, so a timed-out wait
  // only stops this thread's arithmetic, never its barrier arrivals.
  bool ok = true;
  for (int ui = 0; ui < nu; ++ui) {
    const int i = ui * 4 + (cw >> 1);  // stage holding rows 4cw..4cw+3
    const int s = i % NS;
    if (ok && !mbar_wait_sleep(&full[s], (i / NS) & 1)) ok = false;
    float v[V];
#pragma unroll
    for (int q = 0; q < V; ++q) v[q] = 0.f;
    if (ok) {
      const uint8_t* st = stages + (size_t)s * stage_bytes + (size_t)((cw & 1) * 4) * row_bytes;
#pragma unroll
      for (int rr = 0; rr < 4; ++rr) {
#pragma unroll
        for (int k = 0; k < CPL; ++k) {
          const int c = lane + 32 * k;
          if (c < nch) {
            const uint4 w = *reinterpret_cast<const uint4*>(st + (size_t)rr * row_bytes + c * 16);
            const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 f = unpack2<DT>(wv[e]);
#pragma unroll
              for (int b = 0; b < B; ++b) {
                v[rr * B + b] = fmaf(f.x, av[b][k][2 * e], v[rr * B + b]);
                v[rr * B + b] = fmaf(f.y, av[b][k][2 * e + 1], v[rr * B + b]);
              }
            }
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
    const float tot = warp_reduce_transposed<V>(v);
    const int buf = ui & 1;
    if (ok && (lane & ((1 << SH) - 1)) == 0) {
      const int vi = lane >> SH;
      const int rr = vi / B, b = vi % B;
      const int rloc = cw * 4 + rr;  // row within the unit
      const float sv = tot + bias[ui * 32 + rloc];
      const int nrow = (u0 + ui) * 32 + rloc;
      if (p.logits) p.logits[(size_t)b * p.F + nrow] = sv;
      if (sv > p.threshold) atomicOr(&words[buf * B + b], 1u << rloc);
    }
    named_bar_sync(1, kConsumers);
    if (ct < B) {
      p.mask[(size_t)ct * nunits + u0 + ui] = words[buf * B + ct];
      words[buf * B + ct] = 0u;
    }
  }
}

}  // namespace pi
