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

// ------------------------------------------------ both layers, one kernel
// For batch 1-2 both predictor layers run in one grid of two CTAs per SM with
// plain 128-bit register loads, split by a grid-wide barrier.
//   Before the dependency wait: each CTA loads its first W1 rows into
//   registers and asks the L2 for its W2 rows; none of this depends on the
//   previous kernel.
//   Layer 1: row j of W1 goes to CTA j mod G; all 256 threads share each row
//   (thread t holds the 16-byte chunks t, t+256, ... of x and of the row); one
//   block reduction per group of rows gives a_j = relu(W1_j x + b1_j).
//   Grid barrier: every a_j is written.
//   Layer 2: unit u (rows 8u..8u+7 of W2, one mask byte per token) goes to CTA
//   u mod G; warp w of the CTA takes row 8u+w.  The eight bits of a unit meet
//   in shared memory, and each mask byte is written once with a byte store.
struct PredParams {
  const uint8_t* w1;       // [r x d] 16-bit rows
  const float* b1;         // [r] or null
  const uint16_t* x;       // [B x d] 16-bit input (when x_resid is null)
  const float* x_resid;    // [B x d] fp32 residual stream, or null
  uint16_t* x_out;         // [B x d] rounded layer input (written when x_resid)
  float* a;                // [kAReplicas x B x r] fp32
  const uint8_t* w2;       // [F x r] 16-bit rows
  const float* b2;         // [F]
  uint8_t* mask;           // [B x F/8] bytes: the uint32 mask words, byte-addressed
  float* logits;           // [B x F] or null
  uint32_t* bar;           // [2] grid barrier state
  float threshold;
  int d, r, F;
};

constexpr int kPredThreads = 256;
constexpr int kPredWarps = kPredThreads / 32;
constexpr int kPredMaxUnits = 64;  // units of 8 rows per CTA
constexpr int kPredMaxRows1 = 32;  // W1 rows per CTA
// a is written in several copies and CTA c reads copy c mod kAReplicas, so
// the grid's reads right after the barrier spread over more L2 lines
constexpr int kAReplicas = 8;

__host__ __device__ constexpr int pred_p2(int B, int CPL) {
  // layer-2 units in flight per warp: about 96 registers for a and the rows
  return (96 - 8 * B * CPL) / (4 * CPL) < 1 ? 1
         : (96 - 8 * B * CPL) / (4 * CPL) > 8 ? 8
                                               : (96 - 8 * B * CPL) / (4 * CPL);
}

template <int DT, int B, int CPT, int CPL>
__global__ void __launch_bounds__(kPredThreads, 2) k_predict(PredParams p) {
  constexpr int P1 = 8 / CPT;        // W1 rows in flight per thread
  constexpr int V1 = P1 * B;
  constexpr int SH1 = 5 - log2c<V1>();
  constexpr int P2 = pred_p2(B, CPL);
  static_assert(B * CPT <= 4 && B * CPL <= 8, "register budget");
  __shared__ float red1[2][kPredWarps][V1];
  __shared__ float redx[kPredWarps][B];
  __shared__ uint32_t bits[B][kPredMaxUnits];
  __shared__ float bias1[kPredMaxRows1];
  __shared__ float bias2[kPredMaxUnits][kPredWarps];

  const int t = threadIdx.x, lane = t & 31, w = t >> 5;
  const int G = gridDim.x, c = blockIdx.x;
  const int nch1 = p.d / 8;
  const size_t rb1 = (size_t)p.d * 2;
  const int n1 = c < p.r ? (p.r - 1 - c) / G + 1 : 0;  // W1 rows c, c+G, ...
  const int nunits = p.F / 8;
  const int n2 = c < nunits ? (nunits - 1 - c) / G + 1 : 0;  // W2 units c, c+G, ...
  const int nch2 = p.r / 8;
  const size_t rb2 = (size_t)p.r * 2;

  auto load1 = [&](int i, uint4 (&dst)[CPT]) {
    const uint8_t* row = p.w1 + (size_t)(c + i * G) * rb1;
#pragma unroll
    for (int k = 0; k < CPT; ++k) {
      const int u = t + kPredThreads * k;
      dst[k] = (i < n1 && u < nch1) ? ldg_stream(row + (size_t)u * 16) : make_uint4(0, 0, 0, 0);
    }
  };
  uint4 wb[P1][CPT];
#pragma unroll
  for (int q = 0; q < P1; ++q) load1(q, wb[q]);

  for (int e = t; e < B * kPredMaxUnits; e += kPredThreads) (&bits[0][0])[e] = 0u;
  // static biases of this CTA's rows, off the critical path
  if (t < n1) bias1[t] = p.b1 ? p.b1[c + t * G] : 0.f;
  for (int e = t; e < n2 * 8; e += kPredThreads) bias2[e >> 3][e & 7] = p.b2[(size_t)(c + (e >> 3) * G) * 8 + (e & 7)];

  pdl_trigger();
  pdl_wait();  // x (or the residual) comes from the previous kernel

  // this thread's chunks of the layer input, widened to fp32
  float xr[B][CPT][8];
  if (p.x_resid) {
    // x_l = round16(x / sqrt(mean(x^2) + eps)); every CTA forms the same sums
    float4 v[B][CPT][2];
    float ss[B];
#pragma unroll
    for (int b = 0; b < B; ++b) {
      float s2 = 0.f;
#pragma unroll
      for (int k = 0; k < CPT; ++k) {
        const int u = t + kPredThreads * k;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          v[b][k][h] = u < nch1 ? reinterpret_cast<const float4*>(p.x_resid + (size_t)b * p.d)[2 * u + h]
                                : make_float4(0.f, 0.f, 0.f, 0.f);
          s2 = fmaf(v[b][k][h].x, v[b][k][h].x, s2);
          s2 = fmaf(v[b][k][h].y, v[b][k][h].y, s2);
          s2 = fmaf(v[b][k][h].z, v[b][k][h].z, s2);
          s2 = fmaf(v[b][k][h].w, v[b][k][h].w, s2);
        }
      }
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) s2 += __shfl_xor_sync(0xffffffffu, s2, o);
      ss[b] = s2;
    }
    if (lane == 0)
#pragma unroll
      for (int b = 0; b < B; ++b) redx[w][b] = ss[b];
    __syncthreads();
#pragma unroll
    for (int b = 0; b < B; ++b) {
      float tot = 0.f;
#pragma unroll
      for (int i = 0; i < kPredWarps; ++i) tot += redx[i][b];
      const float rms = sqrtf(tot / (float)p.d + kRmsEps);
#pragma unroll
      for (int k = 0; k < CPT; ++k) {
        const int u = t + kPredThreads * k;
        const float f[8] = {v[b][k][0].x, v[b][k][0].y, v[b][k][0].z, v[b][k][0].w,
                            v[b][k][1].x, v[b][k][1].y, v[b][k][1].z, v[b][k][1].w};
        uint32_t pk[4];
#pragma unroll
        for (int e = 0; e < 4; ++e)
          pk[e] = (uint32_t)round16<DT>(f[2 * e] / rms) | ((uint32_t)round16<DT>(f[2 * e + 1] / rms) << 16);
        const uint4 q4 = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        if (u < nch1 && c == 0 && p.x_out)
          reinterpret_cast<uint4*>(p.x_out + (size_t)b * p.d)[u] = q4;
        widen8<DT>(u < nch1 ? q4 : make_uint4(0, 0, 0, 0), xr[b][k]);
      }
    }
  } else {
#pragma unroll
    for (int b = 0; b < B; ++b)
#pragma unroll
      for (int k = 0; k < CPT; ++k) {
        const int u = t + kPredThreads * k;
        const uint4 q4 = u < nch1 ? reinterpret_cast<const uint4*>(p.x + (size_t)b * p.d)[u]
                                  : make_uint4(0, 0, 0, 0);
        widen8<DT>(q4, xr[b][k]);
      }
  }

  // ---- layer 1
  for (int base = 0; base < n1; base += P1) {
    float v[V1];
#pragma unroll
    for (int q = 0; q < P1; ++q) {
#pragma unroll
      for (int b = 0; b < B; ++b) {
        float z = 0.f;
#pragma unroll
        for (int k = 0; k < CPT; ++k) z += dot8<DT>(wb[q][k], xr[b][k]);
        v[q * B + b] = z;
      }
      load1(base + q + P1, wb[q]);
    }
    const float tot = warp_reduce_transposed<V1>(v);
    const int buf = (base / P1) & 1;
    if ((lane & ((1 << SH1) - 1)) == 0) red1[buf][w][lane >> SH1] = tot;
    __syncthreads();
    if (t < V1) {
      const int q = t / B, b = t % B, i = base + q;
      if (i < n1) {
        float z = 0.f;
#pragma unroll
        for (int k = 0; k < kPredWarps; ++k) z += red1[buf][k][t];
        z += bias1[i];
        z = fmaxf(z, 0.f);
#pragma unroll
        for (int rep = 0; rep < kAReplicas; ++rep)
          p.a[((size_t)rep * B + b) * p.r + c + i * G] = z;
      }
    }
  }

  // ---- layer 2: the first rows are requested before the barrier
  auto load2 = [&](int i, uint4 (&dst)[CPL]) {
    const uint8_t* row = p.w2 + ((size_t)(c + i * G) * 8 + w) * rb2;
#pragma unroll
    for (int k = 0; k < CPL; ++k) {
      const int cc = lane + 32 * k;
      dst[k] = (i < n2 && cc < nch2) ? ldg_stream(row + (size_t)cc * 16) : make_uint4(0, 0, 0, 0);
    }
  };
  uint4 wr[P2][CPL];
#pragma unroll
  for (int q = 0; q < P2; ++q) load2(q, wr[q]);

  const bool synced = grid_barrier(p.bar);

  float av[B][CPL][8];
#pragma unroll
  for (int b = 0; b < B; ++b)
#pragma unroll
    for (int k = 0; k < CPL; ++k) {
      const int cc = lane + 32 * k;
      const float4* src =
          reinterpret_cast<const float4*>(p.a + ((size_t)(c % kAReplicas) * B + b) * p.r) + 2 * cc;
      const float4 lo = cc < nch2 ? __ldcg(src) : make_float4(0.f, 0.f, 0.f, 0.f);
      const float4 hi = cc < nch2 ? __ldcg(src + 1) : make_float4(0.f, 0.f, 0.f, 0.f);
      av[b][k][0] = lo.x; av[b][k][1] = lo.y; av[b][k][2] = lo.z; av[b][k][3] = lo.w;
      av[b][k][4] = hi.x; av[b][k][5] = hi.y; av[b][k][6] = hi.z; av[b][k][7] = hi.w;
    }

  for (int base = 0; base < n2; base += P2) {
#pragma unroll
    for (int q = 0; q < P2; ++q) {
      const int i = base + q;
      float v[B];
#pragma unroll
      for (int b = 0; b < B; ++b) v[b] = 0.f;
#pragma unroll
      for (int k = 0; k < CPL; ++k) {
        const uint32_t wv[4] = {wr[q][k].x, wr[q][k].y, wr[q][k].z, wr[q][k].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = unpack2<DT>(wv[e]);
#pragma unroll
          for (int b = 0; b < B; ++b) {
            v[b] = fmaf(f.x, av[b][k][2 * e], v[b]);
            v[b] = fmaf(f.y, av[b][k][2 * e + 1], v[b]);
          }
        }
      }
      load2(i + P2, wr[q]);
#pragma unroll
      for (int b = 0; b < B; ++b)
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) v[b] += __shfl_xor_sync(0xffffffffu, v[b], o);
      if (i < n2 && lane == 0 && synced) {
        const int row = (c + i * G) * 8 + w;
        const float bias = bias2[i][w];
#pragma unroll
        for (int b = 0; b < B; ++b) {
          const float s = v[b] + bias;
          if (p.logits) p.logits[(size_t)b * p.F + row] = s;
          if (s > p.threshold) atomicOr(&bits[b][i], 1u << w);
        }
      }
    }
  }
  __syncthreads();
  for (int e = t; e < B * n2; e += kPredThreads) {
    const int b = e / n2, i = e % n2;
    p.mask[(size_t)b * nunits + c + i * G] = (uint8_t)bits[b][i];
  }
}

}  // namespace pi
