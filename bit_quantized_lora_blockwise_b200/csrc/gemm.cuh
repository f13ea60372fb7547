// Warp-specialised tcgen05 GEMM for sm_100a, with an optional NF4-dequant
// producer for the A operand and an optional low-rank (LoRA) product folded
// into the same TMEM accumulator.
//
//   D[row, col] = sum_k A[row, k] B[col, k]   (+ sum_j A2[row, j] B2[col, j])
//
// The QLoRA layer (intvml.com "DL0087 QLoRA", Figure 1: the NF4 weight is
// dequantized to a bf16 tile just before the matmul and discarded) maps
// onto it with the weight as the 128-row MMA operand A:
//   forward   Y^T[n, m]  = W'[n, :] . X[m, :]   + B^T[n, :] . (s XA)[m, :]
//   backward  dX^T[k, m] = W'^T[k, :] . dY[m, :] + A[k, :] . (s G)[m, :]
// A is rebuilt from the packed codes by "producer" warps that write bf16
// straight into the 128-byte-swizzled shared-memory layout the tensor core
// reads (K-major rows of W for the forward, MN-major for the backward); no
// bf16 copy of W ever reaches global memory. The same kernel, with A and B
// both loaded by TMA and fp32 split-K partials as output, computes the
// skinny adapter products (X A, dY B^T, X^T G, dY^T XA).
//
// Roles (one CTA per SM, persistent over output tiles):
//   warps 0-3  epilogue: TMEM -> registers -> global (lane quadrant = warp)
//   warp 4     TMA issue (one lane)
//   warp 5     TMEM allocation + MMA issue (one lane)
//   warps 6..  dequant producers (NPW warps, in groups of 4 that take turns)
// Pipeline: STAGES shared-memory stages guarded by mbarriers (tma_full,
// deq_full, empty); two TMEM accumulators (tmem_full, tmem_empty) so the
// epilogue of one tile overlaps the mainloop of the next. Every wait is
// bounded (mbar_wait); on a timeout the CTA drains its own copies and MMAs,
// frees TMEM and returns with the device error word set.
#pragma once

#include "codec.cuh"
#include "ptx.cuh"

namespace qlora {

enum : int { A_TMA_K = 0, A_TMA_MN = 1, A_DEQ_K = 2, A_DEQ_MN = 3 };
enum : int { B_TMA_K = 0, B_TMA_MN = 1 };
enum : int { L2_NONE = 0, L2_A_MN = 1, L2_A_K = 2 };  // A2 major-ness (B2 is K-major)
enum : int { EPI_BF16_T = 0, EPI_F32 = 1 };

struct GemmArgs {
  CUtensorMap tm_a;   // A operand (TMA variants)
  CUtensorMap tm_b;   // B operand
  CUtensorMap tm_pk;  // packed NF4 codes (dequant variants)
  CUtensorMap tm_a2;  // low-rank A2
  CUtensorMap tm_b2;  // low-rank B2
  const uint8_t *q;       // 8-bit constant codes (dequant variants)
  const float *scale2;    // second-level scales (dequant variants)
  void *out;              // EPI_BF16_T: bf16 out[col * out_ld + row]; EPI_F32: fp32 partials
  int64_t out_ld;
  int64_t w_kblocks;      // 64-blocks per weight row (K / 64)
  int rows;               // extent of the 128-row MMA dimension
  int cols;               // extent of the BN-column MMA dimension
  int kblocks;            // 64-deep K blocks of the main product
  int splits;             // split-K count (fp32 partials when > 1 or EPI_F32)
  int lora_kblocks;       // 64-deep K blocks of the low-rank product (last split only)
  int w_rows;             // A_DEQ_K: rows of W (N)
  float out_scale;
  float nf4[16];
  float t8[256];
};

template <int BN_, int ASRC_, int BSRC_, int L2_, int EPI_, int STAGES_, int NPW_>
struct GemmCfg {
  static constexpr int BM = 128, BK = 64, BN = BN_;
  static constexpr int ASRC = ASRC_, BSRC = BSRC_, L2 = L2_, EPI = EPI_;
  static constexpr int STAGES = STAGES_, NPW = NPW_;
  static constexpr bool DEQ = ASRC_ >= A_DEQ_K;
  static constexpr bool A_MN = (ASRC_ == A_TMA_MN) || (ASRC_ == A_DEQ_MN);
  static constexpr bool B_MN = BSRC_ == B_TMA_MN;
  static constexpr int NGROUPS = NPW_ >= 4 ? NPW_ / 4 : 1;
  static_assert(!DEQ || (NPW_ % 4 == 0 && NPW_ >= 4), "dequant needs whole producer groups");
  static_assert(BN_ % 16 == 0 && BN_ >= 16 && BN_ <= 256, "MMA N");
  static_assert(!B_MN || BN_ % 64 == 0, "MN-major B needs whole 64-wide chunks");
  static constexpr int A_BYTES = BM * BK * 2;  // 16 KB
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int P_BYTES = DEQ ? 4096 : 0;
  static constexpr int OFF_A = 0;
  static constexpr int OFF_B = OFF_A + STAGES * A_BYTES;
  static constexpr int OFF_P = OFF_B + STAGES * B_BYTES;
  static constexpr int OFF_BAR = OFF_P + STAGES * P_BYTES;
  // barriers: tma_full[S], deq_full[S], empty[S], tmem_full[2], tmem_empty[2], drain
  static constexpr int NBARS = 3 * STAGES + 5;
  static constexpr int OFF_T8 = OFF_BAR + NBARS * 8;
  static constexpr int OFF_MISC = OFF_T8 + 256 * 4;  // tmem base, abort flag
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;  // + alignment slack
  static constexpr int WARPS = 6 + NPW_;
  static constexpr int THREADS = WARPS * 32;
  static constexpr uint32_t TMEM_COLS = (2 * BN <= 32) ? 32 : (2 * BN <= 64) ? 64
                                        : (2 * BN <= 128) ? 128 : (2 * BN <= 256) ? 256 : 512;
  static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");
  static constexpr uint32_t MAIN_TX = B_BYTES + (DEQ ? P_BYTES : A_BYTES);
  static constexpr uint32_t LORA_TX = A_BYTES + B_BYTES;
};

struct TileCoord {
  int row0, col0, split, kb_begin, nmain, nlora;
};

__device__ __forceinline__ TileCoord tile_coord(const GemmArgs &a, int tile, int row_tiles,
                                                int col_tiles, int BN) {
  TileCoord t;
  const int per_split = row_tiles * col_tiles;
  t.split = tile / per_split;
  const int rem = tile - t.split * per_split;
  const int rt = rem / col_tiles;
  const int ct = rem - rt * col_tiles;
  t.row0 = rt * 128;
  t.col0 = ct * BN;
  t.kb_begin = static_cast<int>((static_cast<int64_t>(t.split) * a.kblocks) / a.splits);
  const int kb_end = static_cast<int>((static_cast<int64_t>(t.split + 1) * a.kblocks) / a.splits);
  t.nmain = kb_end - t.kb_begin;
  t.nlora = (t.split == a.splits - 1) ? a.lora_kblocks : 0;
  return t;
}

// Warp-collective bounded wait: every lane waits (each acquires), and the
// warp gives up together if any lane gave up.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int *abort_flag) {
  const bool ok = mbar_wait(bar, parity, abort_flag);
  return __all_sync(0xFFFFFFFFu, ok);
}

template <class C>
__global__ void __launch_bounds__(C::THREADS, 1) qgemm_kernel(const __grid_constant__ GemmArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  const uint32_t bar0 = sbase + C::OFF_BAR;
  auto tma_full = [&](int s) { return bar0 + 8u * s; };
  auto deq_full = [&](int s) { return bar0 + 8u * (C::STAGES + s); };
  auto empty_bar = [&](int s) { return bar0 + 8u * (2 * C::STAGES + s); };
  auto tmem_full = [&](int a) { return bar0 + 8u * (3 * C::STAGES + a); };
  auto tmem_empty = [&](int a) { return bar0 + 8u * (3 * C::STAGES + 2 + a); };
  const uint32_t drain_bar = bar0 + 8u * (3 * C::STAGES + 4);
  float *s_t8 = reinterpret_cast<float *>(smem + C::OFF_T8);
  uint32_t *s_tmem = reinterpret_cast<uint32_t *>(smem + C::OFF_MISC);
  volatile int *s_abort = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(tma_full(s), 1);
      mbar_init(deq_full(s), 4);
      mbar_init(empty_bar(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tmem_full(a), 1);
      mbar_init(tmem_empty(a), 4);
    }
    mbar_init(drain_bar, 1);
    *s_abort = 0;
    fence_barrier_init();
  }
  if (C::DEQ) {
    for (int i = threadIdx.x; i < 256; i += C::THREADS) s_t8[i] = args.t8[i];
  }
  if (warp == 4 && lane == 0) {
    tma_prefetch_desc(&args.tm_b);
    if (!C::DEQ) tma_prefetch_desc(&args.tm_a);
    if (C::DEQ) tma_prefetch_desc(&args.tm_pk);
    if (C::L2 != L2_NONE) {
      tma_prefetch_desc(&args.tm_a2);
      tma_prefetch_desc(&args.tm_b2);
    }
  }
  if (warp == 5) {
    tmem_alloc(smem_u32(s_tmem), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *s_tmem;

  const int row_tiles = (args.rows + 127) / 128;
  const int col_tiles = (args.cols + C::BN - 1) / C::BN;
  const int num_tiles = row_tiles * col_tiles * args.splits;

  if (warp == 4) {
    // ------------------------------------------------------ TMA issue --
    if (lane == 0) {
      uint32_t job = 0;
      for (int tile = blockIdx.x; tile < num_tiles && !*s_abort; tile += gridDim.x) {
        const TileCoord t = tile_coord(args, tile, row_tiles, col_tiles, C::BN);
        const int njobs = t.nmain + t.nlora;
        bool ok = true;
        for (int jj = 0; jj < njobs; ++jj, ++job) {
          const int s = job % C::STAGES;
          const uint32_t par = (job / C::STAGES) & 1u;
          if (!mbar_wait(empty_bar(s), par ^ 1u, s_abort)) { ok = false; break; }
          const uint32_t a_dst = sbase + C::OFF_A + s * C::A_BYTES;
          const uint32_t b_dst = sbase + C::OFF_B + s * C::B_BYTES;
          if (jj < t.nmain) {
            const int kb = t.kb_begin + jj;
            mbar_arrive_expect_tx(tma_full(s), C::MAIN_TX);
            if (C::BSRC == B_TMA_K) {
              tma_load_2d(b_dst, &args.tm_b, tma_full(s), kb * 64, t.col0);
            } else {
#pragma unroll
              for (int c = 0; c < C::BN / 64; ++c)
                tma_load_2d(b_dst + c * 8192, &args.tm_b, tma_full(s), t.col0 + c * 64, kb * 64);
            }
            if (C::ASRC == A_TMA_K) {
              tma_load_2d(a_dst, &args.tm_a, tma_full(s), kb * 64, t.row0);
            } else if (C::ASRC == A_TMA_MN) {
              tma_load_2d(a_dst, &args.tm_a, tma_full(s), t.row0, kb * 64);
              tma_load_2d(a_dst + 8192, &args.tm_a, tma_full(s), t.row0 + 64, kb * 64);
            } else {
              const uint32_t p_dst = sbase + C::OFF_P + s * C::P_BYTES;
              if (C::ASRC == A_DEQ_K)
                tma_load_2d(p_dst, &args.tm_pk, tma_full(s), kb * 32, t.row0);
              else
                tma_load_2d(p_dst, &args.tm_pk, tma_full(s), t.row0 / 2, kb * 64);
            }
          } else {
            const int lk = jj - t.nmain;
            mbar_arrive_expect_tx(tma_full(s), C::LORA_TX);
            tma_load_2d(b_dst, &args.tm_b2, tma_full(s), lk * 64, t.col0);
            if (C::L2 == L2_A_MN) {
              tma_load_2d(a_dst, &args.tm_a2, tma_full(s), t.row0, lk * 64);
              tma_load_2d(a_dst + 8192, &args.tm_a2, tma_full(s), t.row0 + 64, lk * 64);
            } else {
              tma_load_2d(a_dst, &args.tm_a2, tma_full(s), lk * 64, t.row0);
            }
          }
        }
        if (!ok) break;
      }
      // wait for this thread's own copies still in flight (bounded)
      const uint32_t inflight = job < (uint32_t)C::STAGES ? job : (uint32_t)C::STAGES;
      for (uint32_t i = 0; i < inflight; ++i) {
        const uint32_t jb = job - 1 - i;
        const unsigned long long t0 = globaltimer_ns();
        while (!mbar_try_wait(tma_full(jb % C::STAGES), (jb / C::STAGES) & 1u)) {
          if (globaltimer_ns() - t0 > kWaitTimeoutNs) break;
        }
      }
    }
    __syncwarp();
  } else if (warp == 5) {
    // ------------------------------------------------------ MMA issue --
    if (lane == 0) {
      uint32_t job = 0, iter = 0;
      for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++iter) {
        const TileCoord t = tile_coord(args, tile, row_tiles, col_tiles, C::BN);
        const int njobs = t.nmain + t.nlora;
        const int acc = iter & 1;
        if (!mbar_wait(tmem_empty(acc), ((iter >> 1) & 1u) ^ 1u, s_abort)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * C::BN;
        bool ok = true;
        for (int jj = 0; jj < njobs; ++jj, ++job) {
          const int s = job % C::STAGES;
          const uint32_t par = (job / C::STAGES) & 1u;
          if (!mbar_wait(tma_full(s), par, s_abort)) { ok = false; break; }
          if (C::DEQ && !mbar_wait(deq_full(s), par, s_abort)) { ok = false; break; }
          tc_fence_after();
          const bool main_job = jj < t.nmain;
          const bool a_mn = main_job ? C::A_MN : (C::L2 == L2_A_MN);
          const bool b_mn = main_job ? C::B_MN : false;
          const uint32_t idesc = make_idesc_bf16(128, C::BN, a_mn ? 1 : 0, b_mn ? 1 : 0);
          const uint32_t a_addr = sbase + C::OFF_A + s * C::A_BYTES;
          const uint32_t b_addr = sbase + C::OFF_B + s * C::B_BYTES;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ad = a_mn ? smem_desc_sw128(a_addr + kk * 2048, 8192, 1024)
                                     : smem_desc_sw128(a_addr + kk * 32, 16, 1024);
            const uint64_t bd = b_mn ? smem_desc_sw128(b_addr + kk * 2048, 8192, 1024)
                                     : smem_desc_sw128(b_addr + kk * 32, 16, 1024);
            tc_mma_ss(d_tmem, ad, bd, idesc, (jj > 0 || kk > 0) ? 1u : 0u);
          }
          tc_commit(empty_bar(s));
        }
        if (!ok) break;
        tc_commit(tmem_full(acc));
      }
      // all MMAs issued by this thread have completed once drain_bar flips
      tc_commit(drain_bar);
      const unsigned long long t0 = globaltimer_ns();
      while (!mbar_try_wait(drain_bar, 0)) {
        if (globaltimer_ns() - t0 > kWaitTimeoutNs) break;
      }
    }
    __syncwarp();
  } else if (warp < 4) {
    // ------------------------------------------------------- epilogue --
    uint32_t iter = 0;
    const int qrow = warp * 32 + lane;  // TMEM lane of this thread
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++iter) {
      const TileCoord t = tile_coord(args, tile, row_tiles, col_tiles, C::BN);
      const int acc = iter & 1;
      if (!warp_wait(tmem_full(acc), (iter >> 1) & 1u, s_abort)) break;
      tc_fence_after();
      const int row = t.row0 + qrow;
#pragma unroll 1
      for (int ch = 0; ch < C::BN / 32; ++ch) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(tmem_base + ((uint32_t)(warp * 32) << 16) + acc * C::BN + ch * 32, v);
        const int col_base = t.col0 + ch * 32;
        if (C::EPI == EPI_BF16_T) {
          __nv_bfloat16 *o = reinterpret_cast<__nv_bfloat16 *>(args.out);
          if (row < args.rows) {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const int col = col_base + j;
              if (col < args.cols)
                o[static_cast<int64_t>(col) * args.out_ld + row] =
                    __float2bfloat16_rn(__uint_as_float(v[j]) * args.out_scale);
            }
          }
        } else {
          const int64_t rows_pad = static_cast<int64_t>(row_tiles) * 128;
          const int64_t cols_pad = static_cast<int64_t>(col_tiles) * C::BN;
          float4 *o = reinterpret_cast<float4 *>(reinterpret_cast<float *>(args.out) +
                                                 (t.split * rows_pad + row) * cols_pad + col_base);
#pragma unroll
          for (int j = 0; j < 8; ++j)
            o[j] = make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]),
                               __uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3]));
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tmem_empty(acc));
    }
  } else if (C::DEQ) {
    // ------------------------------------------------ dequant producers --
    const int pw = warp - 6;
    const int group = pw >> 2;
    const int p = (pw & 3) * 32 + lane;  // 0..127
    float L[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) L[i] = args.nf4[i];
    uint32_t job = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
      const TileCoord t = tile_coord(args, tile, row_tiles, col_tiles, C::BN);
      const int njobs = t.nmain + t.nlora;
      bool ok = true;
      for (int jj = 0; jj < njobs; ++jj, ++job) {
        if ((int)(job % C::NGROUPS) != group) continue;
        const int s = job % C::STAGES;
        const uint32_t par = (job / C::STAGES) & 1u;
        if (jj < t.nmain) {
          const int kb = t.kb_begin + jj;
          int64_t n, kblk;
          bool valid;
          uint32_t p_off, a_off;
          if (C::ASRC == A_DEQ_K) {
            n = t.row0 + p;
            kblk = kb;
            valid = n < args.w_rows;
            p_off = p * 32;
            a_off = p * 128;
          } else {
            n = static_cast<int64_t>(kb) * 64 + (p & 63);
            kblk = t.row0 / 64 + (p >> 6);
            valid = kblk < args.w_kblocks;
            p_off = (p & 63) * 64 + (p >> 6) * 32;
            a_off = (p >> 6) * 8192 + (p & 63) * 128;
          }
          float cp = 0.0f;
          if (valid) {
            const int64_t b = n * args.w_kblocks + kblk;
            cp = __fmul_rn(s_t8[__ldg(args.q + b)], __ldg(args.scale2 + (b >> 8)));
          }
          if (!warp_wait(empty_bar(s), par ^ 1u, s_abort)) { ok = false; break; }
          if (!warp_wait(tma_full(s), par, s_abort)) { ok = false; break; }
          uint8_t *a_slot = smem + C::OFF_A + s * C::A_BYTES;
          const uint32_t swz = p & 7;
          if (valid) {
            const uint8_t *pk = smem + C::OFF_P + s * C::P_BYTES + p_off;
            const uint4 w0 = *reinterpret_cast<const uint4 *>(pk);
            const uint4 w1 = *reinterpret_cast<const uint4 *>(pk + 16);
            const uint32_t words[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
            const Nf4Planes P = make_planes(L, cp);
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              uint32_t o[4];
              nf4_lookup8(P, words[c], o);
              *reinterpret_cast<uint4 *>(a_slot + a_off + ((c ^ swz) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
            }
          } else {
#pragma unroll
            for (int c = 0; c < 8; ++c)
              *reinterpret_cast<uint4 *>(a_slot + a_off + (c << 4)) = make_uint4(0u, 0u, 0u, 0u);
          }
          fence_proxy_async_smem();
        } else {
          if (!warp_wait(empty_bar(s), par ^ 1u, s_abort)) { ok = false; break; }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(deq_full(s));
      }
      if (!ok) break;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

// ------------------------------------------------------------------------
// Deterministic split-K reduction of fp32 partials [splits][rows_pad][cols_pad]:
//   v = sum over splits in order; out[...] = bf16(v * scale) (and out2 with
//   scale2 when given), row-major [rows, cols] with leading dim ld, or
//   transposed ([cols, rows]) when `transpose`.
__global__ void __launch_bounds__(256) splitk_reduce_kernel(const float *__restrict__ part, int splits,
                                                            int rows, int cols, int64_t rows_pad,
                                                            int64_t cols_pad, float scale,
                                                            __nv_bfloat16 *__restrict__ out, int64_t ld,
                                                            float scale2, __nv_bfloat16 *__restrict__ out2,
                                                            int64_t ld2, int transpose) {
  const int64_t total = static_cast<int64_t>(rows) * cols;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total; i += stride) {
    int64_t r, c;
    if (transpose) {  // consecutive threads -> consecutive rows (contiguous output)
      c = i / rows;
      r = i - c * rows;
    } else {
      r = i / cols;
      c = i - r * cols;
    }
    float v = 0.0f;
    for (int s = 0; s < splits; ++s) v += part[(s * rows_pad + r) * cols_pad + c];
    const int64_t o = transpose ? c * ld + r : r * ld + c;
    out[o] = __float2bfloat16_rn(v * scale);
    if (out2 != nullptr) {
      const int64_t o2 = transpose ? c * ld2 + r : r * ld2 + c;
      out2[o2] = __float2bfloat16_rn(v * scale2);
    }
  }
}

}  // namespace qlora
