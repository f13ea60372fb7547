// Warp-specialised tcgen05 GEMM for sm_100a whose A operand is an NF4
// weight tile dequantized on chip, with the low-rank (LoRA) product folded
// into the same TMEM accumulator.
//
//   D[row, col] = sum_k W'[row, k] B[col, k]  +  sum_j A2[row, j] B2[col, j]
//
// The QLoRA layer (intvml.com "DL0087 QLoRA", Figure 1: the NF4 weight is
// dequantized to a bf16 tile just before the matmul and discarded) maps
// onto it with the weight as the 128-row MMA operand A:
//   forward   Y^T[n, m]  = W'[n, :] . X[m, :]   + B^T[n, :] . (s XA)[m, :]
//   backward  dX^T[k, m] = W'^T[k, :] . dY[m, :] + A[k, :] . (s G)[m, :]
// A is rebuilt from the packed codes by "producer" warps that write bf16
// straight into the 128-byte-swizzled shared-memory layout the tensor core
// reads (K-major rows of W for the forward, MN-major for the backward); no
// bf16 copy of W ever reaches global memory. The token operand (X or dY) and
// the low-rank operands arrive by TMA.
//
// CTA pairs (PAIR = true): a cluster of two CTAs on neighbouring SMs computes
// a 256-row weight tile with the pair form of the MMA (cta_group::2). Each
// CTA decodes its own 128 weight rows into its own A stage and loads half of
// the tile's tokens into its own B stage; the leader (cluster rank 0) issues
// M = 256 MMAs that read both CTAs' stages, and each CTA's TMEM receives its
// own 128 rows over all the tile's tokens. Both CTAs' copies complete on the
// leader's stage barrier (CTA-pair form of the TMA load, no multicast); the
// peer's producers and epilogue arrive on the leader's barriers remotely; the
// leader's commits release the stages and accumulators of both CTAs.
//
// Token stages. On this part a TMA load costs about the same time whether it
// moves 16 KB or 64 KB, so one B stage holds BKB consecutive 64-deep K blocks
// of the CTA's tokens, fetched by one 3-D box (the token operand viewed as
// {64, tokens, K/64}); the MMAs of BKB jobs read it before it is released.
// Low-rank K blocks take one B stage each (two 2-D boxes: B2 and A2).
//
// Token sub-tiles (NTT). Every 64-deep job has fixed costs (a decoded tile
// handed from the producers to the MMA thread, a stage released, barrier
// round trips) that on this part take about as long as the four MMAs of a
// 256-token tile. With NTT = 2 each decoded weight tile feeds the MMAs of two
// 256-token sub-tiles, one TMEM accumulator each (the whole 512 columns), so
// those costs and the decode are spread over twice the FLOPs. The two
// accumulators are then not double-buffered across tiles; instead each has
// its own full/empty barriers, the epilogue drains sub-tile 0 first, and the
// next tile's sub-tile-0 MMAs start while sub-tile 1 is still being drained.
// Each CTA loads NTT x B_ROWS consecutive tokens; accumulator column c of
// sub-tile t holds token col0 + (c / B_ROWS) NTT B_ROWS + t B_ROWS + c % B_ROWS.
//
// Roles (one CTA per SM, persistent over output tiles):
//   warps 0-3  epilogue: TMEM -> registers -> global (lane quadrant = warp)
//   warp 4     TMA issue for the B ring and the low-rank operands (one lane)
//   warp 5     TMEM allocation + MMA issue (one lane of the leader)
//   warp 6     TMA issue for the packed-code ring (one lane)
//   warps 7..  dequant producers (NPW warps, in groups of 4 that take turns)
// Rings (mbarrier-guarded): B (SB stages), dequantized A (SA stages, one per
// 64-deep job), packed codes (SP slots of KSUP jobs; each producer thread
// reads its block's 8-bit constant code and second-level scale from global
// memory one job ahead); two TMEM accumulators (tmem_full, tmem_empty) so the
// epilogue of one tile overlaps the mainloop of the next. Every wait is bounded (mbar_wait); on a
// timeout the CTA drains its own copies and MMAs, frees TMEM and returns with
// the device error word set.
#pragma once

#include "codec.cuh"
#include "ptx.cuh"

namespace qlora {

enum : int { A_DEQ_K = 2, A_DEQ_MN = 3 };
enum : int { L2_A_MN = 1, L2_A_K = 2 };  // A2 major-ness (B2 is K-major)

struct GemmArgs {
  CUtensorMap tm_b;   // token operand viewed as {64, tokens, kdim / 64}: box {64, B_ROWS, BKB}
  CUtensorMap tm_pk;  // packed NF4 codes
  CUtensorMap tm_a2;  // low-rank A2
  CUtensorMap tm_b2;  // low-rank B2 [tokens, r]: box {64, B_ROWS}
  // Output: 16-bit (bf16, or fp16 when f16) out[col * out_ld + row] (the transposed tile).
  void *out;
  int64_t out_ld;
  float *part;             // fp32 partials of split tiles [tail_splits][tail tiles][tile columns][TILE_ROWS]
  unsigned int *counters;  // one per split output tile; zero on entry, left zero
  int rows;               // extent of the weight-row MMA dimension
  int cols;               // extent of the token MMA dimension
  int kblocks;            // 64-deep K blocks of the main product
  // Work units: the first full_tiles tiles whole, then every remaining tile
  // cut either into its NTT token sub-tiles (tail_subtiles = NTT: disjoint
  // outputs, each over the whole K) or into tail_splits K ranges (partials
  // reduced by the last split of a tile to finish, in split order), so that
  // the last, partial round of a persistent grid is spread over more CTAs.
  int full_tiles;
  int tail_splits;
  int tail_subtiles;
  int lora_kblocks;       // 64-deep K blocks of the low-rank product (last split only)
  int f16;                // operands, decoded weight and output are fp16 (else bf16)
  // Block constants, decoded by the producers: c'_b = t8[q_b] * scale2[b / 256]
  // for block b = n * wkb + kb of the row-major weight W [N, wkb * 64].
  const uint8_t *q;
  const float *scale2;
  int64_t wkb;
  float nf4[16];
  float t8[256];
};

template <int BN_, int ASRC_, int L2_, int BKB_, int SB_, int SA_, int SP_, int NPW_, bool PAIR_, int NTT_ = 1>
struct GemmCfg {
  static constexpr int BM = 128, BK = 64, BN = BN_;
  static constexpr int ASRC = ASRC_, L2 = L2_;
  static constexpr int BKB = BKB_, SB = SB_, SA = SA_, SP = SP_, NPW = NPW_;
  static constexpr bool PAIR = PAIR_;
  static constexpr int NTT = NTT_;                 // token sub-tiles (accumulators) per job
  static constexpr int NCTA = PAIR_ ? 2 : 1;       // CTAs per tile
  static constexpr int TILE_ROWS = 128 * NCTA;     // weight rows per tile
  static constexpr int TILE_COLS = BN_ * NTT_;     // tokens per tile
  static constexpr int B_ROWS = BN_ / NCTA;        // tokens of one sub-tile this CTA loads
  static constexpr int CTA_TOK = B_ROWS * NTT_;    // tokens of the tile this CTA loads
  static_assert(NTT_ == 1 || NTT_ == 2, "one or two token sub-tiles");
  static_assert(CTA_TOK <= 256, "a TMA box spans at most 256 tokens");
  static constexpr bool A_MN = ASRC_ == A_DEQ_MN;
  static constexpr int NGROUPS = NPW_ / 4;
  static_assert(NPW_ % 4 == 0 && NPW_ >= 4 && SP_ >= 2, "producer groups of 4 warps and a packed-code ring");
  // (a 16-warp, 3-slot configuration timed out on B200: every producer group
  // needs a slot of its own plus a spare, or the groups wait on each other)
  static_assert(SA_ > NPW_ / 4, "dequantized-tile ring needs more slots than producer groups");
  static_assert(BN_ % 16 == 0 && BN_ >= 16 && BN_ <= 256 && B_ROWS % 8 == 0, "MMA N");
  static_assert(BKB_ >= 1 && BKB_ <= 4, "K blocks per token stage");
  static constexpr int NCHUNK = (BN_ + 31) / 32;  // epilogue chunks of 32 columns (last may hold 16)
  static constexpr int A_BYTES = BM * BK * 2;     // 16 KB
  static constexpr int KB_BYTES = CTA_TOK * BK * 2;  // one K block of this CTA's tokens
  static constexpr int B_BYTES = KB_BYTES * BKB;
  // P slot: the packed codes of KSUP consecutive 64-deep K blocks of the
  // 128-row weight tile (128 contiguous bytes per weight row: forward;
  // 64 bytes of 4 x 64 rows: backward), by TMA, shared by KSUP consecutive
  // MMA jobs. (The block constants come from q and scale2 directly.)
  static constexpr int KSUP = 4;
  static constexpr int PK_BYTES = 4096 * KSUP;
  static constexpr int P_BYTES = PK_BYTES;
  static constexpr int OFF_B = 0;
  static constexpr int OFF_A = OFF_B + SB * B_BYTES;
  static constexpr int OFF_P = OFF_A + SA * A_BYTES;
  static constexpr int OFF_BAR = OFF_P + SP * P_BYTES;
  // b_full[SB] b_empty[SB] a_full[SA] a_empty[SA] p_full[SP] p_empty[SP]
  // tmem_full[2] tmem_empty[2] drain epilogue-group
  static constexpr int NBARS = 2 * SB + 2 * SA + 2 * SP + 6;
  // misc: tmem base, abort flag, last-CTA flag (16 B), the 16 NF4 levels,
  // then the 256-entry 8-bit constant table
  static constexpr int OFF_MISC = ((OFF_BAR + NBARS * 8) + 15) & ~15;
  static constexpr int OFF_T8 = OFF_MISC + 16 + 64;
  static constexpr int SMEM_BYTES = OFF_T8 + 1024;
  static constexpr int WARPS = 7 + NPW_;
  static constexpr int THREADS = WARPS * 32;
  // two accumulators of BN columns: double-buffered tiles (NTT = 1) or the
  // two sub-tiles of one tile (NTT = 2)
  static constexpr uint32_t TMEM_COLS = (2 * BN <= 32) ? 32 : (2 * BN <= 64) ? 64
                                        : (2 * BN <= 128) ? 128 : (2 * BN <= 256) ? 256 : 512;
  static constexpr uint32_t ACC_STRIDE = TMEM_COLS / 2;  // column offset of accumulator 1
  static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");
  // bytes the (leader's) stage barrier expects: both CTAs' copies for a pair
  static constexpr uint32_t MAIN_TX = B_BYTES * NCTA;
  static constexpr uint32_t LORA_TX = (A_BYTES + KB_BYTES) * NCTA;
  static constexpr uint32_t GROUP_ARRIVALS = 4 * NCTA;  // a_full / tmem_empty: 4 warps per CTA
};

struct TileCoord {
  int row0, col0, rc, kb_begin, nmain, nlora;  // rc: (128-row tile, col tile) index
  int split, nsplit, tail;  // K range split of nsplit (1: the whole K); tail: index among the split tiles
  int only;                 // the one token sub-tile this unit computes, or -1 for all
};

// Tile `tile` of a grid of row_tiles x col_tiles tiles of (128 ncta) rows x
// BN columns per split; row0 is the first of this CTA's 128 rows (`rank` in
// the pair).
__device__ __forceinline__ TileCoord tile_coord(const GemmArgs &a, int unit, int row_tiles,
                                                int col_tiles, int tile_cols, int ncta, int rank) {
  TileCoord t;
  int id;  // output tile
  t.only = -1;
  if (unit < a.full_tiles) {
    id = unit;
    t.split = 0;
    t.nsplit = 1;
    t.tail = -1;
  } else if (a.tail_subtiles > 1) {
    const int v = unit - a.full_tiles;
    t.tail = v / a.tail_subtiles;
    t.only = v - t.tail * a.tail_subtiles;
    t.split = 0;
    t.nsplit = 1;
    id = a.full_tiles + t.tail;
  } else {
    const int v = unit - a.full_tiles;
    t.tail = v / a.tail_splits;
    t.split = v - t.tail * a.tail_splits;
    t.nsplit = a.tail_splits;
    id = a.full_tiles + t.tail;
  }
  const int rt = id / col_tiles;
  const int ct = id - rt * col_tiles;
  t.rc = (rt * ncta + rank) * col_tiles + ct;
  t.row0 = (rt * ncta + rank) * 128;
  t.col0 = ct * tile_cols;
  t.kb_begin = static_cast<int>((static_cast<int64_t>(t.split) * a.kblocks) / t.nsplit);
  const int kb_end = static_cast<int>((static_cast<int64_t>(t.split + 1) * a.kblocks) / t.nsplit);
  t.nmain = kb_end - t.kb_begin;
  t.nlora = (t.split == t.nsplit - 1) ? a.lora_kblocks : 0;
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
  const uint32_t epi_bar = bar0 + 8u * (TB + 5);  // the four epilogue warps' group barrier
  uint32_t *s_tmem = reinterpret_cast<uint32_t *>(smem + C::OFF_MISC);
  volatile int *s_abort = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::SB; ++s) {
      mbar_init(b_full(s), 1);
      mbar_init(b_empty(s), 1);
    }
    for (int s = 0; s < C::SA; ++s) {
      mbar_init(a_full(s), C::GROUP_ARRIVALS);
      mbar_init(a_empty(s), 1);
    }
    for (int s = 0; s < C::SP; ++s) {
      mbar_init(p_full(s), 1);
      mbar_init(p_empty(s), 4 * C::KSUP);  // 4 warps per sub-job
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tmem_full(a), 1);
      mbar_init(tmem_empty(a), C::GROUP_ARRIVALS);
    }
    mbar_init(drain_bar, 1);
    mbar_init(epi_bar, 4);
    *s_abort = 0;
    fence_barrier_init();
  }
  if (threadIdx.x < 16) reinterpret_cast<float *>(smem + C::OFF_MISC + 16)[threadIdx.x] = args.nf4[threadIdx.x];
  for (int i = threadIdx.x; i < 256; i += blockDim.x) reinterpret_cast<float *>(smem + C::OFF_T8)[i] = args.t8[i];
  if (warp == 4 && lane == 0) {
    tma_prefetch_desc(&args.tm_b);
    tma_prefetch_desc(&args.tm_a2);
    tma_prefetch_desc(&args.tm_b2);
  }
  if (warp == 6 && lane == 0) tma_prefetch_desc(&args.tm_pk);
  if (warp == 5) {
    if constexpr (C::PAIR) {
      tmem_alloc_pair(smem_u32(s_tmem), C::TMEM_COLS);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(smem_u32(s_tmem), C::TMEM_COLS);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  // a pair: both CTAs' barriers are initialised (and their TMEM allocated)
  // before either CTA's copies, arrivals or commits reach the other
  if constexpr (C::PAIR) cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = *s_tmem;
  // pair rank (0 = leader, which issues the MMAs)
  const uint32_t rank = C::PAIR ? cluster_ctarank() : 0u;
  // Arrivals on barriers the leader waits on. In a pair the arriving thread
  // signals that its own CTA's shared memory (a decoded A half) or TMEM (an
  // accumulator half it has read) is ready; only its own SM's tensor core
  // touches that memory next, so the arrival carries the default CTA-scope
  // release. (A cluster-scope release here cost a third of the kernel's
  // throughput on B200.)
  auto arrive_leader = [&](uint32_t bar) {
    if constexpr (C::PAIR) mbar_arrive_remote(map_cluster(bar, 0u));
    else mbar_arrive(bar);
  };
  auto wait_warp = [&](uint32_t bar, uint32_t par) -> bool {
    return __all_sync(0xFFFFFFFFu, mbar_wait(bar, par, s_abort));
  };
  // Programmatic launch. The kernel before this one in the stream is the
  // call's low-rank launch (X A or dY B^T), and everything before that is
  // complete when this kernel starts (that launch waits for it before it
  // lets this one start). This kernel reads that launch's outputs only in
  // two places: the low-rank operand (the token TMA warp, before its first
  // low-rank stage) and the split-K tile counters it zeroes (the epilogue,
  // before its first counter); everything else (tokens, packed codes and
  // constants, the adapter weights) is an input of the call, so the main K
  // loop runs while that launch is still working. The TMA warp alone lets
  // the next kernel start, and only after its own wait, so a started
  // dependent still implies that this call's earlier launches are complete.

  // tiles of TILE_ROWS weight rows x BN tokens; a pair (cluster) takes every
  // (number of pairs)-th tile
  const int row_tiles = (args.rows + C::TILE_ROWS - 1) / C::TILE_ROWS;
  const int col_tiles = (args.cols + C::TILE_COLS - 1) / C::TILE_COLS;
  const int num_tiles = args.full_tiles + (row_tiles * col_tiles - args.full_tiles) *
                                             (args.tail_subtiles > 1 ? args.tail_subtiles : args.tail_splits);
  const int first_tile = static_cast<int>(blockIdx.x) / C::NCTA;
  const int tile_step = static_cast<int>(gridDim.x) / C::NCTA;
  auto coord = [&](int tile) { return tile_coord(args, tile, row_tiles, col_tiles, C::TILE_COLS, C::NCTA, rank); };

  if (warp == 4) {
    // --------------------------------- TMA: token stages, low-rank operands --
    if (lane == 0) {
      uint32_t job = 0, bs = 0;  // A-ring job and B-ring stage counters
      bool ok = true;
      bool waited = false;
      auto wait_prior = [&]() {
        if (!waited) {
          grid_dep_wait();
          grid_dep_launch();
          waited = true;
        }
      };
      // one stage load: into this CTA's slot, counted on the leader's barrier
      auto load = [&](uint32_t dst, const CUtensorMap *map, uint32_t bar, int x, int y) {
        if constexpr (C::PAIR) tma_load_2d_pair(dst, map, map_cluster(bar, 0u), x, y);
        else tma_load_2d(dst, map, bar, x, y);
      };
      for (int tile = first_tile; ok && tile < num_tiles; tile += tile_step) {
        const TileCoord t = coord(tile);
        const int nbm = (t.nmain + C::BKB - 1) / C::BKB;
        for (int st = 0; st < nbm + t.nlora; ++st, ++bs) {
          const int sb = bs % C::SB;
          if (!mbar_wait(b_empty(sb), ((bs / C::SB) & 1u) ^ 1u, s_abort)) { ok = false; break; }
          const uint32_t b_dst = sbase + C::OFF_B + sb * C::B_BYTES;
          if (st < nbm) {
            // BKB K blocks of this CTA's tokens, one 3-D box
            if (rank == 0) mbar_arrive_expect_tx(b_full(sb), C::MAIN_TX);
            const int kb = t.kb_begin + st * C::BKB;
            const int tok = t.col0 + static_cast<int>(rank) * C::CTA_TOK;
            if constexpr (C::PAIR) tma_load_3d_pair(b_dst, &args.tm_b, map_cluster(b_full(sb), 0u), 0, tok, kb);
            else tma_load_3d(b_dst, &args.tm_b, b_full(sb), 0, tok, kb);
            job += (st + 1 < nbm) ? C::BKB : t.nmain - st * C::BKB;
          } else {
            // low-rank K block: B2 into the stage, A2 into this job's A slot
            wait_prior();  // B2 is the previous launch's output
            const int lk = st - nbm;
            const int sa = job % C::SA;
            if (!mbar_wait(a_empty(sa), ((job / C::SA) & 1u) ^ 1u, s_abort)) { ok = false; break; }
            const uint32_t a_dst = sbase + C::OFF_A + sa * C::A_BYTES;
            if (rank == 0) mbar_arrive_expect_tx(b_full(sb), C::LORA_TX);
            load(b_dst, &args.tm_b2, b_full(sb), lk * 64, t.col0 + static_cast<int>(rank) * C::CTA_TOK);
            if (C::L2 == L2_A_MN) {
              load(a_dst, &args.tm_a2, b_full(sb), t.row0, lk * 64);
              load(a_dst + 8192, &args.tm_a2, b_full(sb), t.row0 + 64, lk * 64);
            } else {
              load(a_dst, &args.tm_a2, b_full(sb), lk * 64, t.row0);
            }
            ++job;
          }
        }
      }
      wait_prior();
      // wait (bounded) for this thread's copies still in flight (a pair's
      // copies complete on the leader's barriers, which count both halves;
      // the peer stays resident until the leader is past this point: the
      // cluster barrier at the end)
      const uint32_t inflight = rank != 0 ? 0u : (bs < (uint32_t)C::SB ? bs : (uint32_t)C::SB);
      for (uint32_t i = 0; i < inflight; ++i) {
        const uint32_t jb = bs - 1 - i;
        const unsigned long long t0 = globaltimer_ns();
        while (!mbar_try_wait(b_full(jb % C::SB), (jb / C::SB) & 1u)) {
          if (globaltimer_ns() - t0 > kWaitTimeoutNs) break;
        }
      }
    }
    __syncwarp();
  } else if (warp == 5) {
    // ------------------------------------------------------ MMA issue --
    // One thread issues every MMA of the CTA (of the pair: the leader's),
    // so this loop is kept lean: the fixed bits of both descriptor layouts
    // and both instruction descriptors are formed once, and each MMA only
    // adds its K offset to the start address field. A pair's MMAs read both
    // CTAs' stages (same offsets), so the leader's barriers count both CTAs'
    // copies and producers, and its commits release the stage in both CTAs
    // (mask 0b11).
    if (lane == 0 && rank == 0) {
      constexpr uint64_t DK = smem_desc_const(16, 1024);    // K-major, 128B swizzle
      constexpr uint64_t DM = smem_desc_const(8192, 1024);  // MN-major, 128B swizzle
      const uint32_t ID_MAIN = idesc_dtype(make_idesc_bf16(C::TILE_ROWS, C::BN, C::A_MN ? 1 : 0, 0), args.f16);
      const uint32_t ID_LORA =
          idesc_dtype(make_idesc_bf16(C::TILE_ROWS, C::BN, C::L2 == L2_A_MN ? 1 : 0, 0), args.f16);
      auto wait_full = [&](uint32_t bar, uint32_t par) -> bool {
        return mbar_try_wait(bar, par) || mbar_wait(bar, par, s_abort);
      };
      auto mma = [&](uint32_t d, uint64_t ad, uint64_t bd, uint32_t id, uint32_t accum) {
        if constexpr (C::PAIR) tc_mma_ss_pair(d, ad, bd, id, accum);
        else tc_mma_ss(d, ad, bd, id, accum);
      };
      auto commit = [&](uint32_t bar) {
        if constexpr (C::PAIR) tc_commit_pair(bar, 0x3);
        else tc_commit(bar);
      };
      const uint32_t a_base = sbase + C::OFF_A, b_base = sbase + C::OFF_B;
      uint32_t job = 0, bs = 0, iter = 0;
      bool ok = true;
      for (int tile = first_tile; ok && tile < num_tiles; tile += tile_step, ++iter) {
        const TileCoord t = coord(tile);
        const int njobs = t.nmain + t.nlora;
        // accumulator use u = iter * NTT + sub-tile: accumulator u & 1, phase u >> 1
        const uint32_t u0 = iter * C::NTT;
        int sa = job % C::SA;
        uint32_t pa = (job / C::SA) & 1u;
        for (int jj = 0; jj < njobs; ++jj, ++job) {
          const bool main_job = jj < t.nmain;
          const int sub = main_job ? jj % C::BKB : 0;  // K block within the token stage
          const bool last_of_stage = !main_job || sub == C::BKB - 1 || jj == t.nmain - 1;
          const int sb = bs % C::SB;
          if (sub == 0 && !wait_full(b_full(sb), (bs / C::SB) & 1u)) { ok = false; break; }
          if (!wait_full(a_full(sa), pa)) { ok = false; break; }
          tc_fence_after();
          const bool a_mn = main_job ? C::A_MN : (C::L2 == L2_A_MN);
          const uint64_t ad = (a_mn ? DM : DK) | (((a_base + sa * C::A_BYTES) >> 4) & 0x3FFFu);
          const uint64_t bd = DK | (((b_base + sb * C::B_BYTES + sub * C::KB_BYTES) >> 4) & 0x3FFFu);
          const uint32_t astep = a_mn ? 2048u >> 4 : 32u >> 4, bstep = 32u >> 4;
          const uint32_t idesc = main_job ? ID_MAIN : ID_LORA;
#pragma unroll
          for (int st = 0; st < C::NTT; ++st) {
            const uint32_t u = u0 + st;
            if (jj == 0) {  // the accumulator's previous tile has been drained
              if (!wait_full(tmem_empty(u & 1u), ((u >> 1) & 1u) ^ 1u)) { ok = false; break; }
              tc_fence_after();
            }
            if (t.only >= 0 && st != t.only) {
              // a sub-tile this unit leaves to another: its accumulator's
              // phases still advance (nothing to drain, nothing written)
              if (jj == njobs - 1) commit(tmem_full(u & 1u));
              continue;
            }
            const uint32_t d_tmem = tmem_base + (u & 1u) * C::ACC_STRIDE;
            const uint64_t bst = bd + ((st * C::B_ROWS * 128) >> 4);  // sub-tile st's tokens of the stage
            mma(d_tmem, ad, bst, idesc, jj > 0 ? 1u : 0u);
            mma(d_tmem, ad + astep, bst + bstep, idesc, 1u);
            mma(d_tmem, ad + 2 * astep, bst + 2 * bstep, idesc, 1u);
            mma(d_tmem, ad + 3 * astep, bst + 3 * bstep, idesc, 1u);
            if (jj == njobs - 1) commit(tmem_full(u & 1u));  // this sub-tile's sum is complete
          }
          if (!ok) break;
          commit(a_empty(sa));
          if (last_of_stage) {
            commit(b_empty(sb));
            ++bs;
          }
          if (++sa == C::SA) { sa = 0; pa ^= 1u; }
        }
      }
      // all MMAs issued by this thread have completed once drain_bar flips
      if constexpr (C::PAIR) tc_commit_pair(drain_bar, 0x1);
      else tc_commit(drain_bar);
      const unsigned long long t0 = globaltimer_ns();
      while (!mbar_try_wait(drain_bar, 0)) {
        if (globaltimer_ns() - t0 > kWaitTimeoutNs) break;
      }
    }
    __syncwarp();
  } else if (warp < 4) {
    // ------------------------------------------------------- epilogue --
    auto qrow_of = [](int w, int l) { return w * 32 + l; };
    // A whole tile: TMEM -> bf16 output directly. A split tile: TMEM -> fp32
    // partial in global memory; the last of the tile's splits to arrive
    // (atomic counter) sums the partials in split order (deterministic) and
    // writes the bf16 output.
    volatile int *s_last = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 8);
    // partial rows are padded to whole 32-column chunks per sub-tile
    constexpr int TILE_PCOLS = C::NTT * C::NCHUNK * 32;
    const int ntail = row_tiles * col_tiles - args.full_tiles;
    // Partial of split sp of tail tile ti, column-major ([column][row]) so
    // that the 32 threads of a warp (32 consecutive rows) store and load 128
    // contiguous bytes: this thread's element of column c is part_col(..)[c * TILE_ROWS].
    auto part_col = [&](int sp, int ti) {
      return args.part + (static_cast<int64_t>(sp) * ntail + ti) * TILE_PCOLS * C::TILE_ROWS + rank * 128 +
             qrow_of(warp, lane);
    };
    uint32_t iter = 0, epi_phase = 0;
    const int qrow = qrow_of(warp, lane);  // TMEM lane of this thread
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
    // out[token][row] for the 32 consecutive tokens from tok (clipped at the
    // last token); each warp store covers 32 consecutive rows
    auto store_out = [&](int row, int tok, const float (&v)[32]) {
      if (row >= args.rows) return;
      const int ncol = args.cols - tok < 32 ? args.cols - tok : 32;
      uint16_t *dst = reinterpret_cast<uint16_t *>(args.out);
      const bool f16 = args.f16 != 0;
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (j < ncol) dst[static_cast<int64_t>(tok + j) * args.out_ld + row] = to_16(v[j], f16);
    };
    bool ok = true;
    for (int tile = first_tile; ok && tile < num_tiles; tile += tile_step, ++iter) {
      const TileCoord t = coord(tile);
      const int row = t.row0 + qrow;
      // first token of chunk ch of sub-tile st (32 columns never straddle the CTA halves)
      auto tok0 = [&](int st, int ch) {
        const int c0 = ch * 32;
        return t.col0 + (c0 / C::B_ROWS) * C::CTA_TOK + st * C::B_ROWS + c0 % C::B_ROWS;
      };
      float *pcol = t.nsplit > 1 ? part_col(t.split, t.tail) : nullptr;
#pragma unroll 1
      for (int st = 0; st < C::NTT; ++st) {
        const uint32_t u = iter * C::NTT + st;
        if (!wait_warp(tmem_full(u & 1u), (u >> 1) & 1u)) { ok = false; break; }
        tc_fence_after();
        if (t.only >= 0 && st != t.only) {  // computed by another unit
          tc_fence_before();
          __syncwarp();
          if (lane == 0) arrive_leader(tmem_empty(u & 1u));
          continue;
        }
        const uint32_t tcol = tmem_base + ((uint32_t)(warp * 32) << 16) + (u & 1u) * C::ACC_STRIDE;
#pragma unroll 1
        for (int ch = 0; ch < C::NCHUNK; ++ch) {
          uint32_t w[32];
          load_chunk(tcol, ch, w);
          if (t.nsplit == 1) {
            float v[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(w[j]);
            store_out(row, tok0(st, ch), v);
          } else {
            float *o = pcol + static_cast<int64_t>((st * C::NCHUNK + ch) * 32) * C::TILE_ROWS;
#pragma unroll
            for (int j = 0; j < 32; ++j) __stcg(o + j * C::TILE_ROWS, __uint_as_float(w[j]));
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) arrive_leader(tmem_empty(u & 1u));  // accumulator free (its partial is in memory)
      }
      if (!ok || t.nsplit == 1) continue;
      grid_dep_wait();  // the tile counters are zeroed by the previous launch
      __threadfence();
      if (!warp_group_sync(epi_bar, epi_phase, s_abort)) { ok = false; continue; }
      if (warp == 0 && lane == 0) {
        const unsigned int prev = atomicAdd(args.counters + t.rc, 1u);
        const int last = prev == static_cast<unsigned int>(t.nsplit - 1);
        if (last) args.counters[t.rc] = 0u;  // every split has arrived: reset for the next use
        *s_last = last;
      }
      if (!warp_group_sync(epi_bar, epi_phase, s_abort)) { ok = false; continue; }
      if (*s_last) {
        __threadfence();
#pragma unroll 1
        for (int pc = 0; pc < C::NTT * C::NCHUNK; ++pc) {
          float v[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = 0.0f;
          for (int sp = 0; sp < t.nsplit; ++sp) {
            const float *src = part_col(sp, t.tail) + static_cast<int64_t>(pc * 32) * C::TILE_ROWS;
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] += __ldcg(src + j * C::TILE_ROWS);
          }
          store_out(row, tok0(pc / C::NCHUNK, pc % C::NCHUNK), v);
        }
      }
    }
  } else if (warp == 6) {
    // ------------------------------------------------ P ring: TMA issue --
    // Runs up to SP superjobs ahead of the producers, gated only by them:
    // the packed codes of the 128 x (64 KSUP) weight tile.
    if (lane == 0) {
      uint32_t ms = 0;  // superjob counter (KSUP main jobs each, per tile)
      bool ok = true;
      for (int tile = first_tile; ok && tile < num_tiles; tile += tile_step) {
        const TileCoord t = coord(tile);
        for (int u = 0; u * C::KSUP < t.nmain; ++u, ++ms) {
          const int sp = ms % C::SP;
          if (!mbar_wait(p_empty(sp), ((ms / C::SP) & 1u) ^ 1u, s_abort)) { ok = false; break; }
          const int kb0 = t.kb_begin + u * C::KSUP;
          const uint32_t p_dst = sbase + C::OFF_P + sp * C::P_BYTES;
          mbar_arrive_expect_tx(p_full(sp), C::P_BYTES);
          if (C::ASRC == A_DEQ_K) tma_load_2d(p_dst, &args.tm_pk, p_full(sp), kb0 * 32, t.row0);
          else tma_load_2d(p_dst, &args.tm_pk, p_full(sp), t.row0 / 2, kb0 * 64);
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
    // the 8-bit code and second-level scale of this thread's block in main
    // job jj of tile t (0 and 0.0 past the weight)
    auto load_consts = [&](const TileCoord &t, int jj, uint32_t &qv, float &sv) {
      int64_t n, kblk;  // W row and 64-block of this thread's codes
      bool valid;
      if (C::ASRC == A_DEQ_K) {
        n = t.row0 + p;
        kblk = t.kb_begin + jj;
        valid = n < args.rows;
      } else {
        n = static_cast<int64_t>(t.kb_begin + jj) * 64 + (p & 63);
        kblk = t.row0 / 64 + (p >> 6);
        valid = kblk < args.wkb;
      }
      qv = 0u;
      sv = 0.0f;
      if (valid) {
        const int64_t b = n * args.wkb + kblk;
        qv = __ldg(args.q + b);
        sv = __ldg(args.scale2 + (b >> 8));
      }
    };
    int pf_jj = -1;  // main job of the current tile whose constants are in pf_q, pf_s
    uint32_t pf_q = 0u;
    float pf_s = 0.0f;
    for (int tile = first_tile; ok && tile < num_tiles; tile += tile_step) {
      const TileCoord t = coord(tile);
      const int njobs = t.nmain + t.nlora;
      pf_jj = -1;
      const int nsup = (t.nmain + C::KSUP - 1) / C::KSUP;
      for (int jj = 0; jj < njobs; ++jj, ++job) {
        const bool main_job = jj < t.nmain;
        if ((int)(job % C::NGROUPS) != group) continue;
        // this thread's block constant for the job, c' = t8[q] * S (the same
        // fp32 product as the dequantization): its code and scale were loaded
        // one of this group's jobs ahead (or here, for a tile's first jobs)
        uint32_t qv = 0u;
        float sv = 0.0f;  // rows past the weight: c' = 0, the rows decode to zeros
        if (main_job) {
          if (pf_jj == jj) {
            qv = pf_q;
            sv = pf_s;
          } else {
            load_consts(t, jj, qv, sv);
          }
          if (jj + C::NGROUPS < t.nmain) {  // this group's next job of the tile
            load_consts(t, jj + C::NGROUPS, pf_q, pf_s);
            pf_jj = jj + C::NGROUPS;
          } else {
            pf_jj = -1;
          }
        }
        const int sa = job % C::SA;
        if (!wait_warp(a_empty(sa), ((job / C::SA) & 1u) ^ 1u)) { ok = false; break; }
        if (main_job) {
          const uint32_t my_ms = ms + jj / C::KSUP;
          const int sub = jj % C::KSUP;
          const int sp = my_ms % C::SP;
          if (!wait_warp(p_full(sp), (my_ms / C::SP) & 1u)) { ok = false; break; }
          const uint8_t *pslot = smem + C::OFF_P + sp * C::P_BYTES;
          // The codes arrive swizzled (TMA 128-byte swizzle on 128-byte rows
          // for the forward, 64-byte swizzle on 64-byte rows for the
          // backward): 16-byte chunk c of a row sits at c ^ (row bits), so
          // the 8 threads of each quarter-warp read 8 different bank groups.
          uint32_t p_off0, p_off1;
          if (C::ASRC == A_DEQ_K) {  // [128 rows][KSUP x 32 B]
            const uint32_t x = p & 7;
            p_off0 = p * (32 * C::KSUP) + (((2 * sub) ^ x) << 4);
            p_off1 = p * (32 * C::KSUP) + (((2 * sub + 1) ^ x) << 4);
          } else {  // [KSUP x 64 rows][2 x 32 B]
            const uint32_t row = sub * 64 + (p & 63), x = (row >> 1) & 3, c0 = 2 * (p >> 6);
            p_off0 = row * 64 + ((c0 ^ x) << 4);
            p_off1 = row * 64 + (((c0 + 1) ^ x) << 4);
          }
          const float cp = __fmul_rn(reinterpret_cast<const float *>(smem + C::OFF_T8)[qv], sv);
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
          const Nf4Planes P = make_planes(L, cp, args.f16 != 0);
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            uint32_t o[4];
            nf4_lookup8(P, words[c], o);
            *reinterpret_cast<uint4 *>(a_slot + a_off + ((c ^ swz) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
          }
          fence_proxy_async_smem();
        }
        __syncwarp();
        if (lane == 0) arrive_leader(a_full(sa));
      }
      ms += nsup;
    }
  }

  tc_fence_before();
  __syncthreads();
  // a pair: neither CTA frees its TMEM or exits while the other may still
  // read its shared memory (the leader's MMAs) or signal its barriers
  if constexpr (C::PAIR) cluster_sync();
  if (warp == 5) {
    tc_fence_after();
    if constexpr (C::PAIR) tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
    else tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

}  // namespace qlora
