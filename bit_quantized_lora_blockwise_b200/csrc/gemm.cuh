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

struct GemmArgs {
  CUtensorMap tm_a;   // A operand (TMA variants)
  CUtensorMap tm_b;   // B operand
  CUtensorMap tm_pk;  // packed NF4 codes (dequant variants)
  CUtensorMap tm_a2;  // low-rank A2
  CUtensorMap tm_b2;  // low-rank B2
  CUtensorMap tm_cp;  // decoded block constants c' [K/64][N] fp32 (dequant variants)
  // Output: bf16 out[row * out_ld + col] (transpose = 0) or
  // out[col * out_ld + row] (transpose = 1), times out_scale; optionally a
  // second copy out2 (same layout, out2_ld) times out2_scale.
  void *out;
  void *out2;
  int64_t out_ld;
  int64_t out2_ld;
  float *part;             // fp32 split-K partials [splits][rows_pad][cols_pad] (splits > 1)
  unsigned int *counters;  // one per output tile; zero on entry, left zero (splits > 1)
  int64_t w_kblocks;      // 64-blocks per weight row (K / 64)
  int rows;               // extent of the 128-row MMA dimension
  int cols;               // extent of the BN-column MMA dimension
  int kblocks;            // 64-deep K blocks of the main product
  int splits;             // split-K count (> 1: partials reduced by the last CTA of a tile)
  int lora_kblocks;       // 64-deep K blocks of the low-rank product (last split only)
  int w_rows;             // A_DEQ_K: rows of W (N)
  float out_scale;
  float out2_scale;
  int transpose;
  float nf4[16];
};

template <int BN_, int ASRC_, int BSRC_, int L2_, int SB_, int SA_, int SP_, int NPW_>
struct GemmCfg {
  static constexpr int BM = 128, BK = 64, BN = BN_;
  static constexpr int ASRC = ASRC_, BSRC = BSRC_, L2 = L2_;
  static constexpr int SB = SB_, SA = SA_, SP = SP_, NPW = NPW_;
  static constexpr bool DEQ = ASRC_ >= A_DEQ_K;
  static constexpr bool A_MN = (ASRC_ == A_TMA_MN) || (ASRC_ == A_DEQ_MN);
  static constexpr bool B_MN = BSRC_ == B_TMA_MN;
  static constexpr int NGROUPS = NPW_ >= 4 ? NPW_ / 4 : 1;
  static_assert(!DEQ || (NPW_ % 4 == 0 && NPW_ >= 4 && SP_ >= 2), "dequant needs producer groups and a P ring");
  static_assert(DEQ || (SA_ == SB_ && SP_ == 0 && NPW_ == 0), "TMA-only A shares the B ring");
  // (a 16-warp, 3-slot configuration timed out on B200: keep a slot per
  // producer group and one spare)
  static_assert(!DEQ || SA_ > NPW_ / 4, "dequantized-tile ring needs more slots than producer groups");
  static_assert(DEQ || L2_ == L2_NONE, "low-rank steps only in the dequant variants");
  static_assert(BN_ % 16 == 0 && BN_ >= 16 && BN_ <= 256, "MMA N");
  static constexpr int NCHUNK = (BN_ + 31) / 32;  // epilogue chunks of 32 columns (last may hold 16)
  static_assert(!B_MN || BN_ % 64 == 0, "MN-major B needs whole 64-wide chunks");
  static constexpr int A_BYTES = BM * BK * 2;  // 16 KB
  static constexpr int B_BYTES = BN * BK * 2;
  // P slot: the packed codes of KSUP consecutive 64-deep K blocks of the
  // 128-row weight tile (128 contiguous bytes per weight row: forward;
  // 64 bytes of 4 x 64 rows: backward), then their 4 x 128 decoded block
  // constants c'; both by TMA, shared by KSUP consecutive MMA jobs.
  static constexpr int KSUP = 4;
  static constexpr int PK_BYTES = 4096 * KSUP;
  static constexpr int P_CP = PK_BYTES;
  static constexpr int P_BYTES = P_CP + 512 * KSUP;
  static constexpr int OFF_B = 0;
  static constexpr int OFF_A = OFF_B + SB * B_BYTES;
  static constexpr int OFF_P = OFF_A + SA * A_BYTES;
  static constexpr int OFF_BAR = OFF_P + SP * P_BYTES;
  // b_full[SB] b_empty[SB] a_full[SA] a_empty[SA] p_full[SP] p_empty[SP]
  // tmem_full[2] tmem_empty[2] drain
  static constexpr int NBARS = 2 * SB + 2 * SA + 2 * SP + 5;
  // misc: tmem base, abort flag, last-CTA flag (16 B), then the 16 NF4 levels
  static constexpr int OFF_MISC = ((OFF_BAR + NBARS * 8) + 15) & ~15;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 64;
  static constexpr int WARPS = DEQ ? 7 + NPW_ : 6;
  static constexpr int THREADS = WARPS * 32;
  static constexpr uint32_t TMEM_COLS = (2 * BN <= 32) ? 32 : (2 * BN <= 64) ? 64
                                        : (2 * BN <= 128) ? 128 : (2 * BN <= 256) ? 256 : 512;
  static constexpr uint32_t ACC_STRIDE = TMEM_COLS / 2;  // column offset of accumulator 1
  static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");
  static constexpr uint32_t MAIN_TX = B_BYTES + (DEQ ? 0 : A_BYTES);
  static constexpr uint32_t LORA_TX = A_BYTES + B_BYTES;
};

struct TileCoord {
  int row0, col0, split, rc, kb_begin, nmain, nlora;  // rc: (row tile, col tile) index
};

__device__ __forceinline__ TileCoord tile_coord(const GemmArgs &a, int tile, int row_tiles,
                                                int col_tiles, int BN) {
  TileCoord t;
  const int per_split = row_tiles * col_tiles;
  t.split = tile / per_split;
  const int rem = tile - t.split * per_split;
  t.rc = rem;
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


template <class C>
__global__ void __launch_bounds__(C::THREADS, 1) qgemm_kernel(const __grid_constant__ GemmArgs args) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = smem_raw;  // 1024-byte aligned: the 128-byte swizzle atoms need it
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  const uint32_t bar0 = sbase + C::OFF_BAR;
  auto b_full = [&](int s) { return bar0 + 8u * s; };
  auto b_empty = [&](int s) { return bar0 + 8u * (C::SB + s); };
  auto a_full = [&](int s) { return bar0 + 8u * (2 * C::SB + s); };
  auto a_empty = [&](int s) { return bar0 + 8u * (2 * C::SB + C::SA + s); };
  auto p_full = [&](int s) { return bar0 + 8u * (2 * C::SB + 2 * C::SA + s); };
  auto p_empty = [&](int s) { return bar0 + 8u * (2 * C::SB + 2 * C::SA + C::SP + s); };
  constexpr int TB = 2 * C::SB + 2 * C::SA + 2 * C::SP;
  auto tmem_full = [&](int a) { return bar0 + 8u * (TB + a); };
  auto tmem_empty = [&](int a) { return bar0 + 8u * (TB + 2 + a); };
  const uint32_t drain_bar = bar0 + 8u * (TB + 4);
  uint32_t *s_tmem = reinterpret_cast<uint32_t *>(smem + C::OFF_MISC);
  volatile int *s_abort = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::SB; ++s) {
      mbar_init(b_full(s), 1);
      mbar_init(b_empty(s), 1);
    }
    for (int s = 0; s < C::SA; ++s) {
      mbar_init(a_full(s), 4);
      mbar_init(a_empty(s), 1);
    }
    for (int s = 0; s < C::SP; ++s) {
      mbar_init(p_full(s), 1);
      mbar_init(p_empty(s), 4 * C::KSUP);  // 4 warps per sub-job
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tmem_full(a), 1);
      mbar_init(tmem_empty(a), 4);
    }
    mbar_init(drain_bar, 1);
    *s_abort = 0;
    fence_barrier_init();
  }
  if (threadIdx.x < 16) reinterpret_cast<float *>(smem + C::OFF_MISC + 16)[threadIdx.x] = args.nf4[threadIdx.x];
  if (warp == 4 && lane == 0) {
    tma_prefetch_desc(&args.tm_b);
    if (!C::DEQ) tma_prefetch_desc(&args.tm_a);
    if (C::L2 != L2_NONE) {
      tma_prefetch_desc(&args.tm_a2);
      tma_prefetch_desc(&args.tm_b2);
    }
  }
  if (C::DEQ && warp == 6 && lane == 0) {
    tma_prefetch_desc(&args.tm_pk);
    tma_prefetch_desc(&args.tm_cp);
  }
  if (warp == 5) {
    tmem_alloc(smem_u32(s_tmem), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *s_tmem;
  // everything above overlaps the previous kernel's tail; its outputs are
  // read only below
  grid_dep_wait();
  grid_dep_launch();

  const int row_tiles = (args.rows + 127) / 128;
  const int col_tiles = (args.cols + C::BN - 1) / C::BN;
  const int num_tiles = row_tiles * col_tiles * args.splits;

  if (warp == 4) {
    // ---------------------------------------- TMA: B ring (and A when TMA) --
    if (lane == 0) {
      uint32_t job = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
        const TileCoord t = tile_coord(args, tile, row_tiles, col_tiles, C::BN);
        const int njobs = t.nmain + t.nlora;
        for (int jj = 0; jj < njobs; ++jj, ++job) {
          const int sb = job % C::SB;
          if (!mbar_wait(b_empty(sb), ((job / C::SB) & 1u) ^ 1u, s_abort)) { ok = false; break; }
          const uint32_t b_dst = sbase + C::OFF_B + sb * C::B_BYTES;
          if (jj < t.nmain) {
            const int kb = t.kb_begin + jj;
            mbar_arrive_expect_tx(b_full(sb), C::MAIN_TX);
            if (C::BSRC == B_TMA_K) {
              tma_load_2d(b_dst, &args.tm_b, b_full(sb), kb * 64, t.col0);
            } else {
#pragma unroll
              for (int c = 0; c < C::BN / 64; ++c)
                tma_load_2d(b_dst + c * 8192, &args.tm_b, b_full(sb), t.col0 + c * 64, kb * 64);
            }
            if (!C::DEQ) {  // A shares the B ring slot index
              const uint32_t a_dst = sbase + C::OFF_A + sb * C::A_BYTES;
              if (C::ASRC == A_TMA_K) {
                tma_load_2d(a_dst, &args.tm_a, b_full(sb), kb * 64, t.row0);
              } else {
                tma_load_2d(a_dst, &args.tm_a, b_full(sb), t.row0, kb * 64);
                tma_load_2d(a_dst + 8192, &args.tm_a, b_full(sb), t.row0 + 64, kb * 64);
              }
            }
          } else {
            // low-rank step: A2 into the A ring slot of this job, B2 into B
            const int lk = jj - t.nmain;
            const int sa = job % C::SA;
            if (!mbar_wait(a_empty(sa), ((job / C::SA) & 1u) ^ 1u, s_abort)) { ok = false; break; }
            const uint32_t a_dst = sbase + C::OFF_A + sa * C::A_BYTES;
            mbar_arrive_expect_tx(b_full(sb), C::LORA_TX);
            tma_load_2d(b_dst, &args.tm_b2, b_full(sb), lk * 64, t.col0);
            if (C::L2 == L2_A_MN) {
              tma_load_2d(a_dst, &args.tm_a2, b_full(sb), t.row0, lk * 64);
              tma_load_2d(a_dst + 8192, &args.tm_a2, b_full(sb), t.row0 + 64, lk * 64);
            } else {
              tma_load_2d(a_dst, &args.tm_a2, b_full(sb), lk * 64, t.row0);
            }
          }
        }
      }
      // wait (bounded) for this thread's copies still in flight
      const uint32_t inflight = job < (uint32_t)C::SB ? job : (uint32_t)C::SB;
      for (uint32_t i = 0; i < inflight; ++i) {
        const uint32_t jb = job - 1 - i;
        const unsigned long long t0 = globaltimer_ns();
        while (!mbar_try_wait(b_full(jb % C::SB), (jb / C::SB) & 1u)) {
          if (globaltimer_ns() - t0 > kWaitTimeoutNs) break;
        }
      }
    }
    __syncwarp();
  } else if (warp == 5) {
    // ------------------------------------------------------ MMA issue --
    // One thread issues every MMA of the CTA, so this loop is kept lean: the
    // fixed bits of both descriptor layouts and both instruction descriptors
    // are formed once, and each MMA only adds its K offset to the start
    // address field.
    if (lane == 0) {
      constexpr uint64_t DK = smem_desc_const(16, 1024);    // K-major, 128B swizzle
      constexpr uint64_t DM = smem_desc_const(8192, 1024);  // MN-major, 128B swizzle
      constexpr uint32_t ID_MAIN = make_idesc_bf16(128, C::BN, C::A_MN ? 1 : 0, C::B_MN ? 1 : 0);
      constexpr uint32_t ID_LORA = make_idesc_bf16(128, C::BN, C::L2 == L2_A_MN ? 1 : 0, 0);
      const uint32_t a_base = sbase + C::OFF_A, b_base = sbase + C::OFF_B;
      uint32_t job = 0, iter = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x, ++iter) {
        const TileCoord t = tile_coord(args, tile, row_tiles, col_tiles, C::BN);
        const int njobs = t.nmain + t.nlora;
        const int acc = iter & 1;
        if (!mbar_wait(tmem_empty(acc), ((iter >> 1) & 1u) ^ 1u, s_abort)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * C::ACC_STRIDE;
        int sb = job % C::SB, sa = C::DEQ ? (int)(job % C::SA) : sb;
        uint32_t pb = (job / C::SB) & 1u, pa = (job / C::SA) & 1u;
        for (int jj = 0; jj < njobs; ++jj, ++job) {
          if (!mbar_try_wait(b_full(sb), pb) && !mbar_wait(b_full(sb), pb, s_abort)) { ok = false; break; }
          if (C::DEQ && !mbar_try_wait(a_full(sa), pa) && !mbar_wait(a_full(sa), pa, s_abort)) { ok = false; break; }
          tc_fence_after();
          const bool main_job = jj < t.nmain;
          const bool a_mn = main_job ? C::A_MN : (C::L2 == L2_A_MN);
          const bool b_mn = main_job && C::B_MN;
          const uint64_t ad = (a_mn ? DM : DK) | (((a_base + sa * C::A_BYTES) >> 4) & 0x3FFFu);
          const uint64_t bd = (b_mn ? DM : DK) | (((b_base + sb * C::B_BYTES) >> 4) & 0x3FFFu);
          const uint32_t astep = a_mn ? 2048u >> 4 : 32u >> 4, bstep = b_mn ? 2048u >> 4 : 32u >> 4;
          const uint32_t idesc = main_job ? ID_MAIN : ID_LORA;
          tc_mma_ss(d_tmem, ad, bd, idesc, jj > 0 ? 1u : 0u);
          tc_mma_ss(d_tmem, ad + astep, bd + bstep, idesc, 1u);
          tc_mma_ss(d_tmem, ad + 2 * astep, bd + 2 * bstep, idesc, 1u);
          tc_mma_ss(d_tmem, ad + 3 * astep, bd + 3 * bstep, idesc, 1u);
          tc_commit(b_empty(sb));
          if (C::DEQ) tc_commit(a_empty(sa));
          if (++sb == C::SB) { sb = 0; pb ^= 1u; }
          if (C::DEQ) {
            if (++sa == C::SA) { sa = 0; pa ^= 1u; }
          } else {
            sa = sb;
          }
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
    // splits == 1: TMEM -> bf16 output directly. splits > 1: TMEM -> fp32
    // partial in global memory; the last of the tile's splits to arrive
    // (atomic counter) sums the partials in split order (deterministic) and
    // writes the bf16 output.
    volatile int *s_last = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 8);
    const int64_t rows_pad = static_cast<int64_t>(row_tiles) * 128;
    // partial rows are padded to whole 32-column chunks per tile
    const int64_t cols_pad = static_cast<int64_t>(col_tiles) * C::NCHUNK * 32;
    uint32_t iter = 0;
    const int qrow = warp * 32 + lane;  // TMEM lane of this thread
    // chunk ch of the accumulator row (32 columns; a 16-column tail is zero-padded)
    auto load_chunk = [&](uint32_t tcol, int ch, uint32_t (&u)[32]) {
      if (C::BN % 32 == 16 && ch == C::NCHUNK - 1) {
        uint32_t h[16];
        tmem_ld_32x32b_x16(tcol + ch * 32, h);
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          u[j] = h[j];
          u[16 + j] = 0u;
        }
      } else {
        tmem_ld_32x32b_x32(tcol + ch * 32, u);
      }
    };
    // col_end: first column past this tile (a 240-wide tile's last chunk
    // must not spill into the next tile)
    auto store_out = [&](int row, int col_base, int col_end, const float (&v)[32]) {
      if (row >= args.rows) return;
      const int lim = col_end < args.cols ? col_end : args.cols;
      const int ncol = lim - col_base < 32 ? lim - col_base : 32;
      for (int o = 0; o < 2; ++o) {
        __nv_bfloat16 *dst = reinterpret_cast<__nv_bfloat16 *>(o ? args.out2 : args.out);
        if (dst == nullptr) continue;
        const float sc = o ? args.out2_scale : args.out_scale;
        const int64_t ld = o ? args.out2_ld : args.out_ld;
        if (args.transpose) {
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (j < ncol) dst[static_cast<int64_t>(col_base + j) * ld + row] = __float2bfloat16_rn(v[j] * sc);
        } else if (ncol == 32) {
          uint32_t w[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) w[j] = pack_bf16x2(v[2 * j] * sc, v[2 * j + 1] * sc);
          uint4 *d4 = reinterpret_cast<uint4 *>(dst + static_cast<int64_t>(row) * ld + col_base);
#pragma unroll
          for (int j = 0; j < 4; ++j) d4[j] = make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (j < ncol) dst[static_cast<int64_t>(row) * ld + col_base + j] = __float2bfloat16_rn(v[j] * sc);
        }
      }
    };
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++iter) {
      const TileCoord t = tile_coord(args, tile, row_tiles, col_tiles, C::BN);
      const int acc = iter & 1;
      if (!warp_wait_all(tmem_full(acc), (iter >> 1) & 1u, s_abort)) break;
      tc_fence_after();
      const int row = t.row0 + qrow;
      const uint32_t tcol = tmem_base + ((uint32_t)(warp * 32) << 16) + acc * C::ACC_STRIDE;
      if (args.splits == 1) {
#pragma unroll 1
        for (int ch = 0; ch < C::NCHUNK; ++ch) {
          uint32_t u[32];
          load_chunk(tcol, ch, u);
          float v[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(u[j]);
          store_out(row, t.col0 + ch * 32, t.col0 + C::BN, v);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(tmem_empty(acc));
        continue;
      }
      float *prow = args.part + (static_cast<int64_t>(t.split) * rows_pad + row) * cols_pad +
                    (t.col0 / C::BN) * (C::NCHUNK * 32);
#pragma unroll 1
      for (int ch = 0; ch < C::NCHUNK; ++ch) {
        uint32_t u[32];
        load_chunk(tcol, ch, u);
        float4 *o = reinterpret_cast<float4 *>(prow + ch * 32);
#pragma unroll
        for (int j = 0; j < 8; ++j)
          o[j] = make_float4(__uint_as_float(u[4 * j]), __uint_as_float(u[4 * j + 1]),
                             __uint_as_float(u[4 * j + 2]), __uint_as_float(u[4 * j + 3]));
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tmem_empty(acc));  // accumulator free: partial is in memory
      __threadfence();
      named_bar_sync(1, 128);
      if (warp == 0 && lane == 0) {
        const unsigned int prev = atomicAdd(args.counters + t.rc, 1u);
        const int last = prev == static_cast<unsigned int>(args.splits - 1);
        if (last) args.counters[t.rc] = 0u;  // every split has arrived: reset for the next use
        *s_last = last;
      }
      named_bar_sync(1, 128);
      if (*s_last) {
        __threadfence();
#pragma unroll 1
        for (int ch = 0; ch < C::NCHUNK; ++ch) {
          float v[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = 0.0f;
          for (int sp = 0; sp < args.splits; ++sp) {
            const float4 *src = reinterpret_cast<const float4 *>(
                args.part + (static_cast<int64_t>(sp) * rows_pad + row) * cols_pad +
                (t.col0 / C::BN) * (C::NCHUNK * 32) + ch * 32);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const float4 x = __ldcg(src + j);
              v[4 * j] += x.x;
              v[4 * j + 1] += x.y;
              v[4 * j + 2] += x.z;
              v[4 * j + 3] += x.w;
            }
          }
          store_out(row, t.col0 + ch * 32, t.col0 + C::BN, v);
        }
      }
    }
  } else if constexpr (C::DEQ) {
   if (warp == 6) {
    // ------------------------------------------------ P ring: TMA issue --
    // Runs up to SP main K blocks ahead of the producers, gated only by them:
    // the packed codes of the 128 x 64 weight tile and its 128 decoded block
    // constants (c' is block-major, so they are one contiguous 512-byte row
    // for the forward and two 256-byte rows for the backward).
    if (lane == 0) {
      uint32_t ms = 0;  // superjob counter (KSUP main jobs each, per tile)
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
        const TileCoord t = tile_coord(args, tile, row_tiles, col_tiles, C::BN);
        for (int u = 0; u * C::KSUP < t.nmain; ++u, ++ms) {
          const int sp = ms % C::SP;
          if (!mbar_wait(p_empty(sp), ((ms / C::SP) & 1u) ^ 1u, s_abort)) { ok = false; break; }
          const int kb0 = t.kb_begin + u * C::KSUP;
          const uint32_t p_dst = sbase + C::OFF_P + sp * C::P_BYTES;
          mbar_arrive_expect_tx(p_full(sp), C::P_BYTES);
          if (C::ASRC == A_DEQ_K) {
            tma_load_2d(p_dst, &args.tm_pk, p_full(sp), kb0 * 32, t.row0);
            tma_load_2d(p_dst + C::P_CP, &args.tm_cp, p_full(sp), t.row0, kb0);
          } else {
            tma_load_2d(p_dst, &args.tm_pk, p_full(sp), t.row0 / 2, kb0 * 64);
            tma_load_2d(p_dst + C::P_CP, &args.tm_cp, p_full(sp), kb0 * 64, t.row0 / 64);
          }
        }
      }
      // wait (bounded) for this thread's own copies still in flight
      const uint32_t inflight = ms < (uint32_t)C::SP ? ms : (uint32_t)C::SP;
      for (uint32_t i = 0; i < inflight; ++i) {
        const uint32_t jb = ms - 1 - i;
        const unsigned long long t0 = globaltimer_ns();
        while (!mbar_try_wait(p_full(jb % C::SP), (jb / C::SP) & 1u)) {
          if (globaltimer_ns() - t0 > kWaitTimeoutNs) break;
        }
      }
    }
    __syncwarp();
   } else {
    // ------------------------------------------------ dequant producers --
    const int pw = warp - 7;
    const int group = pw >> 2;
    const int p = (pw & 3) * 32 + lane;  // 0..127: the tile row this thread decodes
    const uint32_t a_off = (C::ASRC == A_DEQ_K) ? p * 128 : (p >> 6) * 8192 + (p & 63) * 128;
    const uint32_t swz = p & 7;
    uint32_t job = 0, ms = 0;  // ms: superjob counter at the start of the tile
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
      const TileCoord t = tile_coord(args, tile, row_tiles, col_tiles, C::BN);
      const int njobs = t.nmain + t.nlora;
      const int nsup = (t.nmain + C::KSUP - 1) / C::KSUP;
      for (int jj = 0; jj < njobs; ++jj, ++job) {
        const bool main_job = jj < t.nmain;
        if ((int)(job % C::NGROUPS) != group) continue;
        const int sa = job % C::SA;
        if (!warp_wait_all(a_empty(sa), ((job / C::SA) & 1u) ^ 1u, s_abort)) { ok = false; break; }
        if (main_job) {
          const uint32_t my_ms = ms + jj / C::KSUP;
          const int sub = jj % C::KSUP;
          const int sp = my_ms % C::SP;
          if (!warp_wait_all(p_full(sp), (my_ms / C::SP) & 1u, s_abort)) { ok = false; break; }
          const uint8_t *pslot = smem + C::OFF_P + sp * C::P_BYTES;
          // The codes arrive swizzled (TMA 128-byte swizzle on 128-byte rows
          // for the forward, 64-byte swizzle on 64-byte rows for the
          // backward): 16-byte chunk c of a row sits at c ^ (row bits), so
          // the 8 threads of each quarter-warp read 8 different bank groups.
          uint32_t p_off0, p_off1, c_idx;
          if (C::ASRC == A_DEQ_K) {  // [128 rows][KSUP x 32 B], c' [KSUP][128]
            const uint32_t x = p & 7;
            p_off0 = p * (32 * C::KSUP) + (((2 * sub) ^ x) << 4);
            p_off1 = p * (32 * C::KSUP) + (((2 * sub + 1) ^ x) << 4);
            c_idx = sub * 128 + p;
          } else {  // [KSUP x 64 rows][2 x 32 B], c' [2][KSUP x 64]
            const uint32_t row = sub * 64 + (p & 63), x = (row >> 1) & 3, c0 = 2 * (p >> 6);
            p_off0 = row * 64 + ((c0 ^ x) << 4);
            p_off1 = row * 64 + (((c0 + 1) ^ x) << 4);
            c_idx = (p >> 6) * (64 * C::KSUP) + sub * 64 + (p & 63);
          }
          const float cp = reinterpret_cast<const float *>(pslot + C::P_CP)[c_idx];
          const uint4 w0 = *reinterpret_cast<const uint4 *>(pslot + p_off0);
          const uint4 w1 = *reinterpret_cast<const uint4 *>(pslot + p_off1);
          __syncwarp();
          if (lane == 0) {  // this sub-job's share of the slot is consumed
            // a short last superjob releases the missing sub-jobs' shares too
            const int nsub = t.nmain - (jj / C::KSUP) * C::KSUP;
            const int extra = (jj == t.nmain - 1 && nsub < C::KSUP) ? C::KSUP - nsub : 0;
            for (int e = 0; e <= extra; ++e) mbar_arrive(p_empty(sp));
          }
          uint8_t *a_slot = smem + C::OFF_A + sa * C::A_BYTES;
          // out-of-range rows decode with c' = 0 -> zeros
          const uint32_t words[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
          float L[16];  // NF4 levels, re-read each job (shared-memory broadcast) to spare registers
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float4 l4 = reinterpret_cast<const float4 *>(smem + C::OFF_MISC + 16)[i];
            L[4 * i] = l4.x;
            L[4 * i + 1] = l4.y;
            L[4 * i + 2] = l4.z;
            L[4 * i + 3] = l4.w;
          }
          const Nf4Planes P = make_planes(L, cp);
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            uint32_t o[4];
            nf4_lookup8(P, words[c], o);
            *reinterpret_cast<uint4 *>(a_slot + a_off + ((c ^ swz) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
          }
          fence_proxy_async_smem();
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(a_full(sa));
      }
      ms += nsup;
    }
   }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

}  // namespace qlora
