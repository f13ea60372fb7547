// Rank-r adapter products of the QLoRA layer on tcgen05 (sm_100a):
//   X A (forward, before the fused GEMM), dY B^T, X^T G and dY^T (X A)
//   (backward) — out[rows, r] = scale * sum_k Aop[row, k] Bop[j, k].
// The adapters are trainable and only they receive gradients (intvml.com
// "DL0087 QLoRA", component 4; Figure 1, dashed path).
//
// The reduction dimension is long (K, N or M tokens) and the output thin
// (r columns), so K is split across the CTAs of a thread-block cluster (one
// cluster per 128-row tile, up to 8 CTAs). Each CTA streams its K range
// through a TMA ring into a TMEM accumulator, parks its fp32 partial in its
// own shared memory, and after a cluster barrier every CTA sums one slice of
// rows over all the cluster's partials through distributed shared memory,
// in rank order (deterministic), and writes the bf16 result (optionally a
// second copy with another scale, optionally transposed). No global
// partials, no counters, one launch.
//
// Roles: warp 0 TMA, warp 1 TMEM + MMA issue, warps 4-7 TMEM readout (lane
// quadrant = warp - 4); all 8 warps take part in the cluster reduction.
#pragma once

#include "codec.cuh"
#include "ptx.cuh"

namespace qlora {

// One product of the launch.
struct SkinnyProblem {
  CUtensorMap tm_a;  // A operand: K-major box {64, 128} or MN-major 64x64 chunks
  CUtensorMap tm_b;  // B operand: K-major box {64, BN} or MN-major 64x64 chunks
  void *out;         // bf16 [rows, cols] (ld out_ld) or transposed [cols, rows]
  void *out2;        // optional second output, same layout
  int64_t out_ld, out2_ld;
  float out_scale, out2_scale;
  int transpose;
  int rows;     // extent of the 128-row MMA dimension
  int cols;     // r
  int kblocks;  // 64-deep K blocks in total
};

struct SkinnyArgs {
  // Up to two independent products of the same operand layouts in one
  // launch: CTAs [0, prob0_ctas) take prob[0], the next ones prob[1].
  SkinnyProblem prob[2];
  int prob0_ctas;
  int splits;   // CTAs per cluster (1, 2, 4 or 8), each taking a K range
  unsigned int *zero_words;  // optional: words CTA 0 sets to zero (tile counters of the next kernel)
  int nzero;
  int early;  // 1: neither operand is written by the kernel just before this one in the stream, so the
              // first ring stages may be loaded before waiting for that kernel (programmatic launch)
  int late;   // 1: every operand is complete when this launch starts and nothing it writes is touched by
              // the kernel before it, so the whole product runs without waiting for that kernel; each
              // thread waits for it only before exiting, so this grid still completes after it
  int f16;   // operands and outputs are fp16 (else bf16)
};

template <int BN_, bool A_MN_, bool B_MN_, int STAGES_>
struct SkinnyCfg {
  static constexpr int BN = BN_, STAGES = STAGES_;
  static constexpr bool A_MN = A_MN_, B_MN = B_MN_;
  static_assert(BN_ % 64 == 0 && BN_ <= 256, "rank tile");
  static constexpr int A_BYTES = 128 * 64 * 2;
  static constexpr int B_BYTES = BN_ * 64 * 2;
  static constexpr int OFF_A = 0;
  static constexpr int OFF_B = STAGES_ * A_BYTES;
  static constexpr int OFF_BAR = OFF_B + STAGES_ * B_BYTES;
  static constexpr int NBARS = 2 * STAGES_ + 2;  // full[S], empty[S], tmem_full, drain
  static constexpr int OFF_MISC = OFF_BAR + NBARS * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16;
  static constexpr int THREADS = 256;
  static constexpr uint32_t TMEM_COLS = BN_ <= 64 ? 64 : (BN_ <= 128 ? 128 : 256);
  static constexpr int PART_LD = BN_ + 4;  // fp32 per partial row (16-byte pad against bank conflicts)
  static_assert(128 * PART_LD * 4 <= OFF_BAR, "the partial reuses the ring");
  static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");
  static constexpr uint32_t TX = A_BYTES + B_BYTES;
};

template <class C>
__global__ void __launch_bounds__(C::THREADS, 1) skinny_kernel(const __grid_constant__ SkinnyArgs args) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = smem_raw;  // 1024-byte aligned: the 128-byte swizzle atoms need it
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t bar0 = sbase + C::OFF_BAR;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (C::STAGES + s); };
  const uint32_t tmem_full = bar0 + 8u * (2 * C::STAGES);
  const uint32_t drain_bar = bar0 + 8u * (2 * C::STAGES + 1);
  uint32_t *s_tmem = reinterpret_cast<uint32_t *>(smem + C::OFF_MISC);
  volatile int *s_abort = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);

  const int splits = args.splits;
  const int pi = static_cast<int>(blockIdx.x) >= args.prob0_ctas ? 1 : 0;
  const SkinnyProblem &P = args.prob[pi];
  const int local_block = static_cast<int>(blockIdx.x) - (pi ? args.prob0_ctas : 0);
  const uint32_t rank = splits > 1 ? cluster_ctarank() : 0u;
  const int tile = local_block / splits;
  const int row0 = tile * 128;
  const int kb_begin = static_cast<int>((static_cast<int64_t>(rank) * P.kblocks) / splits);
  const int kb_end = static_cast<int>((static_cast<int64_t>(rank + 1) * P.kblocks) / splits);
  const int nk = kb_end - kb_begin;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    mbar_init(tmem_full, 1);
    mbar_init(drain_bar, 1);
    *s_abort = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&P.tm_a);
    tma_prefetch_desc(&P.tm_b);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(s_tmem), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *s_tmem;
  // producer state: stages issued so far (the first ring's worth may go out
  // ahead of the wait for the previous kernel, see SkinnyArgs::early)
  int issued = 0;
  auto issue = [&](int j) {
    const int s = j % C::STAGES;
    const int kb = kb_begin + j;
    const uint32_t a_dst = sbase + C::OFF_A + s * C::A_BYTES;
    const uint32_t b_dst = sbase + C::OFF_B + s * C::B_BYTES;
    mbar_arrive_expect_tx(full_bar(s), C::TX);
    if (C::A_MN) {
      tma_load_2d(a_dst, &P.tm_a, full_bar(s), row0, kb * 64);
      tma_load_2d(a_dst + 8192, &P.tm_a, full_bar(s), row0 + 64, kb * 64);
    } else {
      tma_load_2d(a_dst, &P.tm_a, full_bar(s), kb * 64, row0);
    }
    if (C::B_MN) {
#pragma unroll
      for (int c = 0; c < C::BN / 64; ++c) tma_load_2d(b_dst + c * 8192, &P.tm_b, full_bar(s), c * 64, kb * 64);
    } else {
      tma_load_2d(b_dst, &P.tm_b, full_bar(s), kb * 64, 0);
    }
  };
  if (args.early && !args.late && warp == 0 && lane == 0)
    for (; issued < nk && issued < C::STAGES; ++issued) issue(issued);
  if (!args.late) grid_dep_wait();
  grid_dep_launch();
  if (blockIdx.x == 0)
    for (int i = threadIdx.x; i < args.nzero; i += blockDim.x) args.zero_words[i] = 0u;

  if (warp == 0) {
    if (lane == 0) {
      for (; issued < nk; ++issued) {
        const int s = issued % C::STAGES;
        if (!mbar_wait(empty_bar(s), ((issued / C::STAGES) & 1u) ^ 1u, s_abort)) break;
        issue(issued);
      }
      // wait (bounded) for this thread's copies still in flight
      const int inflight = issued < C::STAGES ? issued : C::STAGES;
      for (int i = 0; i < inflight; ++i) {
        const int jb = issued - 1 - i;
        const unsigned long long t0 = globaltimer_ns();
        while (!mbar_try_wait(full_bar(jb % C::STAGES), (jb / C::STAGES) & 1u)) {
          if (globaltimer_ns() - t0 > kWaitTimeoutNs) break;
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_dtype(make_idesc_bf16(128, C::BN, C::A_MN ? 1 : 0, C::B_MN ? 1 : 0), args.f16);
      bool ok = true;
      for (int j = 0; j < nk; ++j) {
        const int s = j % C::STAGES;
        if (!mbar_wait(full_bar(s), (j / C::STAGES) & 1u, s_abort)) { ok = false; break; }
        tc_fence_after();
        const uint32_t a_addr = sbase + C::OFF_A + s * C::A_BYTES;
        const uint32_t b_addr = sbase + C::OFF_B + s * C::B_BYTES;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t ad = C::A_MN ? smem_desc_sw128(a_addr + kk * 2048, 8192, 1024)
                                      : smem_desc_sw128(a_addr + kk * 32, 16, 1024);
          const uint64_t bd = C::B_MN ? smem_desc_sw128(b_addr + kk * 2048, 8192, 1024)
                                      : smem_desc_sw128(b_addr + kk * 32, 16, 1024);
          tc_mma_ss(tmem_base, ad, bd, idesc, (j > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(empty_bar(s));
      }
      if (ok) tc_commit(tmem_full);
      tc_commit(drain_bar);
      const unsigned long long t0 = globaltimer_ns();
      while (!mbar_try_wait(drain_bar, 0)) {
        if (globaltimer_ns() - t0 > kWaitTimeoutNs) break;
      }
    }
    __syncwarp();
  } else if (warp >= 4) {
    // TMEM -> this CTA's fp32 partial in shared memory (the ring is idle now)
    const int q = warp - 4;
    const bool ok = warp_wait_all(tmem_full, 0, s_abort);
    tc_fence_after();
    float *part = reinterpret_cast<float *>(smem);
    const int lrow = q * 32 + lane;
#pragma unroll 1
    for (int ch = 0; ch < C::BN / 32; ++ch) {
      uint32_t u[32];
      if (ok && nk > 0) {
        tmem_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(q * 32) << 16) + ch * 32, u);
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) u[j] = 0u;
      }
      float4 *dst = reinterpret_cast<float4 *>(part + lrow * C::PART_LD + ch * 32);
#pragma unroll
      for (int j = 0; j < 8; ++j)
        dst[j] = make_float4(__uint_as_float(u[4 * j]), __uint_as_float(u[4 * j + 1]),
                             __uint_as_float(u[4 * j + 2]), __uint_as_float(u[4 * j + 3]));
    }
    tc_fence_before();
  }

  __syncthreads();
  if (splits > 1) cluster_sync();  // every partial of the cluster is in place

  // Reduce this CTA's slice of rows over the cluster's partials, rank order.
  {
    const int R = 128 / splits;
    const int c4n = C::BN / 4;  // float4 per row
    const int units = R * c4n;
    const uint32_t part_addr = sbase;
    for (int u = threadIdx.x; u < units; u += C::THREADS) {
      int lr, c4;
      if (P.transpose) {  // consecutive threads -> consecutive rows (coalesced transposed store)
        c4 = u / R;
        lr = u - c4 * R;
      } else {  // consecutive threads -> consecutive columns
        lr = u / c4n;
        c4 = u - lr * c4n;
      }
      const int lrow = static_cast<int>(rank) * R + lr;
      const uint32_t off = static_cast<uint32_t>((lrow * C::PART_LD + c4 * 4) * 4);
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (splits > 1) {
        // all peers' loads in flight at once, then summed in rank order
        float4 x[8];
#pragma unroll
        for (int sp = 0; sp < 8; ++sp)
          if (sp < splits) x[sp] = ld_cluster_f4(map_cluster(part_addr + off, sp));
#pragma unroll
        for (int sp = 0; sp < 8; ++sp)
          if (sp < splits) {
            v.x += x[sp].x;
            v.y += x[sp].y;
            v.z += x[sp].z;
            v.w += x[sp].w;
          }
      } else {
        v = *reinterpret_cast<const float4 *>(smem + off);
      }
      const int row = row0 + lrow;
      if (row >= P.rows) continue;
      const float vv[4] = {v.x, v.y, v.z, v.w};
      for (int o = 0; o < 2; ++o) {
        uint16_t *dst = reinterpret_cast<uint16_t *>(o ? P.out2 : P.out);
        if (dst == nullptr) continue;
        const float sc = o ? P.out2_scale : P.out_scale;
        const int64_t ld = o ? P.out2_ld : P.out_ld;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int col = c4 * 4 + e;
          if (col >= P.cols) continue;
          const int64_t idx = P.transpose ? static_cast<int64_t>(col) * ld + row
                                             : static_cast<int64_t>(row) * ld + col;
          dst[idx] = to_16(vv[e] * sc, args.f16 != 0);
        }
      }
    }
  }
  if (splits > 1) cluster_sync();  // peers are done reading this CTA's partial

  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
  if (args.late) grid_dep_wait();
}

}  // namespace qlora
