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
// memory) on operands that the tensor memory accelerator gathers straight
// from HBM into 128-byte-swizzled shared memory:
//   - weight rows: cp.async.bulk.tensor .tile::gather4 (four neuron ids per
//     instruction, 64 elements = 128 bytes of each row);
//   - tokens (up) and H (down): ordinary 2-D tensor tiles, rows past the batch
//     filled with zeros by the copy engine.
// One thread issues the copies, one thread the MMAs; four warps read the
// accumulator out of tensor memory (tcgen05.ld) for the epilogue.
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
// Four rows (r0..r3) of a 2-D tensor, box {64 elements, 1 row}, into 512
// contiguous bytes of shared memory; completion counted on *bar.
__device__ __forceinline__ void tma_gather4(void* dst, const CUtensorMap* tm, int col, int r0,
                                            int r1, int r2, int r3, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cta.global.tile::gather4.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3, %4, %5, %6}], [%7];" ::"r"(smem_u32(dst)),
      "l"(tm), "r"(col), "r"(r0), "r"(r1), "r"(r2), "r"(r3), "r"(smem_u32(bar))
      : "memory");
}
// One box of a 2-D tensor at (c0 = inner coordinate, c1 = row).
__device__ __forceinline__ void tma_load2d(void* dst, const CUtensorMap* tm, int c0, int c1,
                                           uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
      "l"(tm), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}

// ---------------------------------------------------------------- kernels
constexpr int kUmmaThreads = 192;  // warp 0 copies, warp 1 MMAs, warps 2-5 epilogue
constexpr int kUmmaM = 128;        // neuron rows (up) / output columns (down) per tile
constexpr int kUmmaK = 64;         // contraction elements per stage (one 128-byte row)

struct UmmaParams {
  const int32_t* idx;      // neuron list (first *count entries)
  const int32_t* count;
  const float* bias;       // up: b_up (ReLU, Squared-ReLU) or b_gate (ReGLU), or null
  uint16_t* hh;            // [B x F] 16-bit hi part of H (token-major)
  uint16_t* hl;            // [B x F] 16-bit lo part
  float* part;             // down: [gridDim.y x B x d] partial y
  int d, F, B;
};

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

// Gathered up projection + activation.  One CTA per tile of 128 listed
// neurons (tiles past the device-side count exit at once); the contraction
// runs over d in stages of 64.  DT: 0 fp16, 1 bf16 weights and tokens.
// ACT: 0 ReLU, 1 ReGLU (gate rows in tm_a, up rows in tm_a2), 2 Squared-ReLU.
// N: tokens per MMA (the batch rounded up to a multiple of 16).
template <int DT, int ACT, int N, int NS>
__global__ void __launch_bounds__(kUmmaThreads, 1)
    k_umma_up(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_a2,
              const __grid_constant__ CUtensorMap tm_x, UmmaParams p) {
  constexpr int NMAT = ACT == 1 ? 2 : 1;
  constexpr int ABYTES = kUmmaM * kUmmaK * 2;  // 16 KB per matrix
  constexpr int STAGE = umma_up_stage<NMAT, N>();
  constexpr uint32_t NCOL = NMAT * N <= 32 ? 32 : NMAT * N <= 64 ? 64 : NMAT * N <= 128 ? 128 : 256;
  constexpr uint32_t IDESC = idesc_f16<DT, kUmmaM, N, 0, 0>();
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
  int K = *p.count;
  K = K < 0 ? 0 : (K > p.F ? p.F : K);
  const int k0 = blockIdx.x * kUmmaM;
  if (k0 >= K) return;  // whole CTA
  const int rows = min(kUmmaM, K - k0);
  if (t < kUmmaM) {
    int id = t < rows ? p.idx[k0 + t] : -1;
    if (t < rows && (id < 0 || id >= p.F)) {
      set_error(kErrBadIndex);
      id = -1;
    }
    ids[t] = id;
    bias_s[t] = (id >= 0 && p.bias) ? p.bias[id] : 0.f;
  }
  if (t == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
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
  const int nst = p.d / kUmmaK;

  if (warp == 0) {
    if (lane == 0) {  // copy engine feeder
      for (int i = 0; i < nst; ++i) {
        const int s = i % NS;
        if (i >= NS && !mbar_wait(&empty[s], ((i / NS) - 1) & 1)) break;
        uint8_t* st = smem + (size_t)s * STAGE;
        mbar_arrive_expect_tx(&full[s], STAGE);
#pragma unroll 1
        for (int q = 0; q < kUmmaM / 4; ++q) {
          const int r0 = max(ids[4 * q], 0), r1 = max(ids[4 * q + 1], 0);
          const int r2 = max(ids[4 * q + 2], 0), r3 = max(ids[4 * q + 3], 0);
          tma_gather4(st + 512 * q, &tm_a, i * kUmmaK, r0, r1, r2, r3, &full[s]);
          if constexpr (NMAT == 2)
            tma_gather4(st + ABYTES + 512 * q, &tm_a2, i * kUmmaK, r0, r1, r2, r3, &full[s]);
        }
        tma_load2d(st + NMAT * ABYTES, &tm_x, i * kUmmaK, 0, &full[s]);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {  // MMA issuer
      for (int i = 0; i < nst; ++i) {
        const int s = i % NS;
        if (!mbar_wait(&full[s], (i / NS) & 1)) break;
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
    // epilogue: warp w reads tensor-memory lanes 32 (w % 4) .. + 31 (neurons)
    const int quad = warp & 3;
    const int m = quad * 32 + lane;
    const bool ok = mbar_wait_sleep(&done, 0);
    tc_fence_after();
    const int k = k0 + m;
    const int id = ids[m];
    const float bias = bias_s[m];
#pragma unroll
    for (int c0 = 0; c0 < N; c0 += 8) {
      uint32_t ra[8], ru[8];
      tmem_ld8(tmem + ((uint32_t)(quad * 32) << 16) + c0, ra);
      if constexpr (NMAT == 2) tmem_ld8(tmem + ((uint32_t)(quad * 32) << 16) + N + c0, ru);
      tmem_wait_ld();
      if (k < p.F) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int n = c0 + j;
          if (n < p.B) {
            float h = 0.f;
            if (ok && id >= 0) {
              const float r = fmaxf(__uint_as_float(ra[j]) + bias, 0.f);
              h = ACT == 1 ? r * __uint_as_float(ru[j]) : ACT == 2 ? r * r : r;
            }
            const uint16_t hi = to16<DT>(h);
            const float fh = from16<DT>(hi);
            if (DT == 0 && isinf(fh)) set_error(kErrRange);
            p.hh[(size_t)n * p.F + k] = hi;
            p.hl[(size_t)n * p.F + k] = to16<DT>(h - fh);
          }
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

// Gathered down projection.  Grid (d / 128 column tiles, S neuron slices);
// CTA (c, s) sums the neuron positions of slice s (stages of 64) into the
// 128 x N accumulator of columns [128c, 128c + 128) and writes it to
// part[s].  Positions past the list hold H = 0 (the up kernel writes zeros
// up to the next multiple of 128), and their rows are gathered from row 0.
template <int DT, int N, int NS>
__global__ void __launch_bounds__(kUmmaThreads, 1)
    k_umma_down(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_hh,
                const __grid_constant__ CUtensorMap tm_hl, UmmaParams p) {
  constexpr int ABYTES = kUmmaM * kUmmaK * 2;  // 2 column atoms of 64 neurons x 128 B
  constexpr int BBYTES = N * kUmmaK * 2;
  constexpr int STAGE = umma_down_stage<N>();
  constexpr uint32_t NCOL = N <= 32 ? 32 : N <= 64 ? 64 : N <= 128 ? 128 : 256;
  constexpr uint32_t IDESC = idesc_f16<DT, kUmmaM, N, 1, 0>();
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  __shared__ uint64_t full[NS], empty[NS], done;
  __shared__ uint32_t tmem_base;

  pdl_wait();
  pdl_trigger();
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
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
      mbar_init(&full[s], 1);
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
    // copy engine feeder: the whole warp reads the stage's 64 neuron ids
    // (two per lane, the next stage's while this one's copies are issued)
    auto ids_of = [&](int i, int& a, int& b) {
      const int kp = (st0 + i) * kUmmaK + 2 * lane;
      a = kp < K ? p.idx[kp] : 0;
      b = kp + 1 < K ? p.idx[kp + 1] : 0;
      a = (a < 0 || a >= p.F) ? 0 : a;  // flagged by the up kernel; its H is 0
      b = (b < 0 || b >= p.F) ? 0 : b;
    };
    int na = 0, nb = 0;
    if (nst > 0) ids_of(0, na, nb);
    for (int i = 0; i < nst; ++i) {
      const int s = i % NS;
      const int ca = na, cb = nb;
      if (i + 1 < nst) ids_of(i + 1, na, nb);
      bool ok = true;
      if (lane == 0) {
        if (i >= NS && !mbar_wait(&empty[s], ((i / NS) - 1) & 1)) ok = false;
        if (ok) mbar_arrive_expect_tx(&full[s], STAGE);
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      uint8_t* st = smem + (size_t)s * STAGE;
#pragma unroll 1
      for (int q = 0; q < kUmmaK / 4; ++q) {  // neurons 4q .. 4q+3 of the stage
        const int r0 = __shfl_sync(0xffffffffu, ca, 2 * q);
        const int r1 = __shfl_sync(0xffffffffu, cb, 2 * q);
        const int r2 = __shfl_sync(0xffffffffu, ca, 2 * q + 1);
        const int r3 = __shfl_sync(0xffffffffu, cb, 2 * q + 1);
        if (lane == 0) {
          tma_gather4(st + 512 * q, &tm_w, col0, r0, r1, r2, r3, &full[s]);
          tma_gather4(st + ABYTES / 2 + 512 * q, &tm_w, col0 + 64, r0, r1, r2, r3, &full[s]);
        }
      }
      if (lane == 0) {
        tma_load2d(st + ABYTES, &tm_hh, (st0 + i) * kUmmaK, 0, &full[s]);
        tma_load2d(st + ABYTES + BBYTES, &tm_hl, (st0 + i) * kUmmaK, 0, &full[s]);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {  // MMA issuer
      for (int i = 0; i < nst; ++i) {
        const int s = i % NS;
        if (!mbar_wait(&full[s], (i / NS) & 1)) break;
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
  } else {
    const int quad = warp & 3;
    const int c = col0 + quad * 32 + lane;  // output column of this lane
    const bool ok = nst == 0 || mbar_wait_sleep(&done, 0);
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
        if (n < p.B && c < p.d)
          p.part[((size_t)blockIdx.y * p.B + n) * p.d + c] =
              (nst > 0 && ok) ? __uint_as_float(r[j]) : 0.f;
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

}  // namespace pi
