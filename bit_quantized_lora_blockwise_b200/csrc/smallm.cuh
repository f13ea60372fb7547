// Few-token forward: Y = X W'^T + B^T-term for M <= 16 tokens, a stream of
// the packed weight with the dequantization done in registers.
//
// The forward of one QLoRA linear (intvml.com "DL0087 QLoRA: 4-bit Quantized
// LoRA", opening paragraph and Figure 1): the base weight is stored as NF4
// codes with double-quantized block constants and is dequantized to bf16
// just before it is multiplied. With a few tokens the layer reads 0.516
// bytes of packed weight per parameter and does 2 M flops with it; what
// bounds it is the HBM stream and the integer work of the decode (about 21
// byte-permute and logic operations per 8 codes), not the tensor cores.
//
// Data path. One producer warp keeps a ring of shared-memory stages full
// with TMA: a stage is one unit's packed codes (256 rows x 128 bytes, one
// 32 KB box, 128-byte swizzle) plus the matching activations (X for the
// unit's 256 K, at most 16 tokens). Sixteen compute warps (one 16-row tile
// each) read their codes from the stage with 16-byte shared loads, decode
// them in registers with a per-block bf16 table and feed warp-level
// 16x8x16 tensor-core MMAs. The block constants (8-bit code and
// second-level scale) are loaded by the compute threads two units ahead.
// Decoupling the stream from the decode keeps five or six units (160-200 KB
// per SM) in flight, so the integer pipe, not memory latency, sets the rate.
//
// Work split. Rows of W come in bands of 256, K in chunks of 256 (four
// quantization blocks). The (band, chunk) units, band-major, are divided
// evenly among a persistent grid (stream-K): a CTA runs a contiguous range
// of units. The pieces of a band computed by different CTAs are parked in
// fp32 slots (at most two per CTA: the band its range starts in and the one
// it ends in); the CTA whose piece completes a band (band counter) sums the
// slots in CTA order, so the result does not depend on timing, and no CTA
// ever waits for another one to be scheduled.
//
// Register fragments. In an m16n8k16 MMA, lane (g, t) = (lane / 4, lane % 4)
// holds A elements (rows g and g+8, logical k 2t, 2t+1, 2t+8, 2t+9) and B
// elements (the same k, token column g). Any bijection between logical and
// physical k that A and B share gives the same sum, so lane t takes the
// whole quantization block t of the chunk: in MMA step (u, h) its logical k
// pairs map to physical k 64t + 8u + 4h + {0,1} and {2,3}. One thread thus
// decodes 64 consecutive codes of a row with one per-block bf16 table, and
// reads the matching 8 bf16 of X with one 16-byte shared-memory load.
#pragma once

#include "codec.cuh"
#include "ptx.cuh"

namespace qlora {

struct SmallmArgs {
  CUtensorMap tm_x;          // X [M, K] bf16 viewed as {64, K/64, M}; box {64, 4, 8 NT}, 128B swizzle
  CUtensorMap tm_w;          // packed [N, K/2] u8; box {128, 256}, 128B swizzle
  const uint8_t *q;          // [N K / 64] 8-bit block-constant codes
  const float *scale2;       // [ceil(N K / 64 / 256)] second-level scales
  const uint16_t *B;         // [r, N] (16-bit: bf16, or fp16 in the fp16 build)
  const uint16_t *xas;       // [M, r] = 16-bit((alpha / r) X A)
  uint16_t *Y;               // [M, N]
  float *part;               // partial slots: [grid][2][16 warps][NT][32 lanes][4]
  unsigned int *counters;    // one per band, zero on entry (left zero): pieces parked
  int64_t N, K;
  int M, r;
  int kc;     // 256-deep K chunks (the last may hold fewer than 4 blocks)
  int units;  // bands * kc
  CodecTables tabs;
};

template <int NT_>
struct SmallmCfg {
  static constexpr int NT = NT_;                 // 8-token MMA column tiles
  static constexpr int WARPS = 16;               // compute warps, one 16-row tile each
  static constexpr int BAND = 16 * WARPS;        // rows of W per band
  static constexpr int THREADS = WARPS * 32;     // lane 0 of warp 0 also issues the stage copies
  static constexpr int XR = 8 * NT;              // token rows per stage
  static constexpr int W_BYTES = BAND * 128;     // [256 rows][128 bytes = 256 codes]
  static constexpr int X_BYTES = 4 * XR * 128;   // [XR tokens][4 blocks][64 bf16]
  static constexpr int STAGE = W_BYTES + X_BYTES;
  static constexpr int SX = NT == 1 ? 6 : 5;     // stages
  static constexpr int OFF_BAR = SX * STAGE;
  // full[SX] empty[SX], then the CTA's group barrier (one arrival per warp)
  static constexpr int OFF_T8 = OFF_BAR + (2 * SX + 2) * 8;
  static constexpr int OFF_MISC = OFF_T8 + 256 * 4;  // abort flag, two completed-band flags
  static constexpr int SMEM_BYTES = OFF_MISC + 16;
  static constexpr int SLOT_FLOATS = WARPS * NT * 32 * 4;
  static_assert(W_BYTES % 1024 == 0 && X_BYTES % 1024 == 0, "stages keep the 1024-byte swizzle alignment");
  static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");
};

// CTA that owns unit u when `units` units are split evenly over `grid` CTAs
// (CTA i runs [floor(i units / grid), floor((i+1) units / grid))).
__host__ __device__ __forceinline__ int smallm_cta_of(int64_t u, int64_t units, int64_t grid) {
  return static_cast<int>(((u + 1) * grid - 1) / units);
}
__host__ __device__ __forceinline__ int smallm_unit_begin(int64_t cta, int64_t units, int64_t grid) {
  return static_cast<int>(cta * units / grid);
}

template <int NT, bool F16>
__global__ void __launch_bounds__(SmallmCfg<NT>::THREADS, 1) smallm_kernel(const __grid_constant__ SmallmArgs a) {
  using C = SmallmCfg<NT>;
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float *s_t8 = reinterpret_cast<float *>(smem + C::OFF_T8);
  volatile int *s_abort = reinterpret_cast<volatile int *>(smem + C::OFF_MISC);
  auto full_bar = [&](int s) { return sbase + C::OFF_BAR + 8u * s; };
  auto empty_bar = [&](int s) { return sbase + C::OFF_BAR + 8u * (C::SX + s); };
  const uint32_t group_bar = sbase + C::OFF_BAR + 8u * (2 * C::SX);

  const int grid = gridDim.x;
  const int u_begin = smallm_unit_begin(blockIdx.x, a.units, grid);
  const int u_end = smallm_unit_begin(blockIdx.x + 1, a.units, grid);
  const int nunits = u_end - u_begin;

  // Stage copies (lane 0 of warp 0): unit j goes to stage j % SX once every
  // warp has released unit j - SX; its codes (one box) and activations (one
  // box) are counted on the stage's full barrier. Before unit i is consumed
  // its copy must be issued (waiting for the slowest warp if needed); later
  // ones are issued when their stage is already free. X and the packed
  // weight are inputs of this call, so the copies need no wait on the launch
  // before.
  int issued = 0, is_band = u_begin / a.kc, is_c = u_begin - (u_begin / a.kc) * a.kc;
  auto issue = [&](int i) {
    while (issued < nunits && issued < i + C::SX) {
      const int j = issued, st = j % C::SX;
      if (j >= C::SX) {
        const uint32_t par = ((j / C::SX) - 1) & 1u;
        if (j == i) {
          if (!mbar_wait_spin(empty_bar(st), par, s_abort)) return;
        } else if (!mbar_try_wait(empty_bar(st), par)) {
          return;
        }
      }
      const uint32_t dst = sbase + st * C::STAGE;
      mbar_arrive_expect_tx(full_bar(st), C::STAGE);
      tma_load_2d(dst, &a.tm_w, full_bar(st), is_c * 128, is_band * C::BAND);
      tma_load_3d(dst + C::W_BYTES, &a.tm_x, full_bar(st), 0, is_c * 4, 0);
      if (++is_c == a.kc) {
        is_c = 0;
        ++is_band;
      }
      ++issued;
    }
  };
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::SX; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), C::WARPS);
    }
    mbar_init(group_bar, C::WARPS);
    *s_abort = 0;
    fence_barrier_init();
    tma_prefetch_desc(&a.tm_w);
    tma_prefetch_desc(&a.tm_x);
    issue(0);  // the first SX stages go out before anything else
  }
  for (int i = threadIdx.x; i < 256; i += blockDim.x) s_t8[i] = a.tabs.t8[i];
  __syncthreads();

  // ------------------------------------------------------ compute warps --
  const int g = lane >> 2, t = lane & 3;
  const int64_t kb_total = a.K / 64;

  // This lane's block constants for one unit (rows g and g + 8 of the warp's
  // tile, block t of the chunk), loaded two units ahead of their use.
  struct Consts {
    uint32_t q[2];
    float s[2];
  };
  int ld_band = u_begin / a.kc, ld_c = u_begin - (u_begin / a.kc) * a.kc;
  auto load_consts = [&](Consts &f) {
    const int64_t row = static_cast<int64_t>(ld_band) * C::BAND + warp * 16 + g;
    const int64_t kb = static_cast<int64_t>(ld_c) * 4 + t;
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      const bool ok = row + 8 * rr < a.N && kb < kb_total;
      const int64_t bi = (row + 8 * rr) * kb_total + kb;
      f.q[rr] = ok ? __ldg(a.q + bi) : 0u;
      f.s[rr] = ok ? __ldg(a.scale2 + (bi >> 8)) : 0.0f;  // c' = 0: the block contributes zeros
    }
    if (++ld_c == a.kc) {
      ld_c = 0;
      ++ld_band;
    }
  };

  float acc[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[nt][e] = 0.0f;

  // Epilogue of a band whose base sum is complete in acc: + B^T[n, :] .
  // xas[m, :] as 16-deep MMA steps, then bf16 Y. The operands of the first
  // 64 ranks are loaded ahead (lora_load), so their latency can hide behind
  // a wait.
  struct LoraFrag {
    uint32_t af[4][4];
    uint32_t bf[4][NT][2];
  };
  auto lora_load = [&](int64_t n0, int j00, LoraFrag &L) {
    const uint16_t *Bh = reinterpret_cast<const uint16_t *>(a.B);
    auto bval = [&](int j, int64_t n) -> uint32_t { return j < a.r ? Bh[static_cast<int64_t>(j) * a.N + n] : 0u; };
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int ja = j00 + 16 * q + 2 * t, jb = ja + 8;
      L.af[q][0] = bval(ja, n0 + g) | (bval(ja + 1, n0 + g) << 16);
      L.af[q][1] = bval(ja, n0 + g + 8) | (bval(ja + 1, n0 + g + 8) << 16);
      L.af[q][2] = bval(jb, n0 + g) | (bval(jb + 1, n0 + g) << 16);
      L.af[q][3] = bval(jb, n0 + g + 8) | (bval(jb + 1, n0 + g + 8) << 16);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int m = 8 * nt + g;
        const uint32_t *xr = reinterpret_cast<const uint32_t *>(a.xas + static_cast<int64_t>(m) * a.r);
        L.bf[q][nt][0] = (m < a.M && ja < a.r) ? xr[ja >> 1] : 0u;
        L.bf[q][nt][1] = (m < a.M && jb < a.r) ? xr[jb >> 1] : 0u;
      }
    }
  };
  auto lora_apply = [&](const LoraFrag &L) {
#pragma unroll
    for (int q = 0; q < 4; ++q)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
        mma_16816<F16>(acc[nt], L.af[q][0], L.af[q][1], L.af[q][2], L.af[q][3], L.bf[q][nt][0], L.bf[q][nt][1]);
  };
  auto band_row0 = [&](int band) { return static_cast<int64_t>(band) * C::BAND + warp * 16; };
  auto store_y = [&](int64_t n0) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int m = 8 * nt + 2 * t + (e & 1);
        const int64_t n = n0 + g + 8 * (e >> 1);
        if (m < a.M) a.Y[static_cast<int64_t>(m) * a.N + n] = to_16(acc[nt][e], F16);
      }
  };
  // after the stream (registers free): first 64 ranks preloaded
  auto epilogue = [&](int band, const LoraFrag &L0) {
    const int64_t n0 = band_row0(band);
    if (n0 >= a.N) return;
    lora_apply(L0);
    for (int j00 = 64; j00 < a.r; j00 += 64) {
      LoraFrag L;
      lora_load(n0, j00, L);
      lora_apply(L);
    }
    store_y(n0);
  };
  // inside the stream (the next unit's loads hold registers): one 16-rank
  // step at a time
  auto epilogue_lean = [&](int band) {
    const int64_t n0 = band_row0(band);
    if (n0 >= a.N) return;
    const uint16_t *Bh = reinterpret_cast<const uint16_t *>(a.B);
    auto bval = [&](int j, int64_t n) -> uint32_t { return j < a.r ? Bh[static_cast<int64_t>(j) * a.N + n] : 0u; };
#pragma unroll 1
    for (int j0 = 0; j0 < a.r; j0 += 16) {
      const int ja = j0 + 2 * t, jb = ja + 8;
      const uint32_t a0 = bval(ja, n0 + g) | (bval(ja + 1, n0 + g) << 16);
      const uint32_t a1 = bval(ja, n0 + g + 8) | (bval(ja + 1, n0 + g + 8) << 16);
      const uint32_t a2 = bval(jb, n0 + g) | (bval(jb + 1, n0 + g) << 16);
      const uint32_t a3 = bval(jb, n0 + g + 8) | (bval(jb + 1, n0 + g + 8) << 16);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int m = 8 * nt + g;
        const uint32_t *xr = reinterpret_cast<const uint32_t *>(a.xas + static_cast<int64_t>(m) * a.r);
        const uint32_t b0 = (m < a.M && ja < a.r) ? xr[ja >> 1] : 0u;
        const uint32_t b1 = (m < a.M && jb < a.r) ? xr[jb >> 1] : 0u;
        mma_16816<F16>(acc[nt], a0, a1, a2, a3, b0, b1);
      }
    }
    store_y(n0);
  };
  // Partial slots of CTA `cta`: 0 holds the piece of the band its range
  // starts in (when an earlier CTA started that band), 1 the piece of the
  // band its range ends in (when later CTAs finish that band).
  auto slot_ptr = [&](int cta, int which) {
    return reinterpret_cast<float4 *>(a.part + (static_cast<size_t>(cta) * 2 + which) * C::SLOT_FLOATS) +
           warp * NT * 32 + lane;
  };

  bool waited = false;
  int first_band = -1;  // band whose later piece this CTA parked in slot 0
  int last_band = -1;   // band whose first piece this CTA parked in slot 1

  // Shared-memory addresses of this lane's data in stage 0. Codes: rows g
  // and g + 8 of the warp's tile, 16-byte chunks 2t and 2t + 1 of the row's
  // 128 bytes, at chunk ^ (row & 7) (row & 7 = g) under the 128-byte
  // swizzle. Activations: token g, block t, 16-byte chunk u at u ^ (4g + t) & 7.
  const uint32_t wrow = sbase + static_cast<uint32_t>((warp * 16 + g) * 128);
  const uint32_t wc0 = static_cast<uint32_t>(((2 * t) ^ g) << 4);
  const uint32_t wc1 = static_cast<uint32_t>(((2 * t + 1) ^ g) << 4);
  const uint32_t swz16 = static_cast<uint32_t>(((4 * g + t) & 7) << 4);
  const uint32_t xrow = sbase + C::W_BYTES + static_cast<uint32_t>((4 * g + t) * 128);
  int cur_band = u_begin / a.kc, cur_c = u_begin - (u_begin / a.kc) * a.kc, piece0 = u_begin;
  // Decode one unit's codes into MMA fragments and accumulate; then
  // release its stage and close the piece if a band ends.
  auto run_unit = [&](int i, const Consts &f) -> bool {
    const float cp0 = __fmul_rn(s_t8[f.q[0]], f.s[0]);
    const float cp1 = __fmul_rn(s_t8[f.q[1]], f.s[1]);
    const int s = i % C::SX;
    if (warp == 0 && lane == 0) issue(i);
    __syncwarp();
    if (!__all_sync(0xFFFFFFFFu, mbar_wait_spin(full_bar(s), (i / C::SX) & 1u, s_abort))) return false;
    const bool rows_here = static_cast<int64_t>(cur_band) * C::BAND + warp * 16 < a.N;
    if (rows_here) {
      const Nf4Planes P0 = make_planes(a.tabs.nf4, cp0, F16);
      const Nf4Planes P1 = make_planes(a.tabs.nf4, cp1, F16);
      const uint32_t ws = wrow + s * C::STAGE;
      const uint4 r0a = lds_16B(ws + wc0), r0b = lds_16B(ws + wc1);
      const uint4 r1a = lds_16B(ws + 8 * 128 + wc0), r1b = lds_16B(ws + 8 * 128 + wc1);
      const uint32_t w0[8] = {r0a.x, r0a.y, r0a.z, r0a.w, r0b.x, r0b.y, r0b.z, r0b.w};
      const uint32_t w1[8] = {r1a.x, r1a.y, r1a.z, r1a.w, r1b.x, r1b.y, r1b.z, r1b.w};
      const uint32_t xs = xrow + s * C::STAGE;
#pragma unroll
      for (int uu = 0; uu < 8; ++uu) {
        uint32_t o0[4], o1[4];
        nf4_lookup8(P0, w0[uu], o0);
        nf4_lookup8(P1, w1[uu], o1);
        const uint32_t xa = xs | ((static_cast<uint32_t>(uu) << 4) ^ swz16);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const uint4 xv = lds_16B(xa + nt * (8 * 4 * 128));
          mma_16816<F16>(acc[nt], o0[0], o1[0], o0[1], o1[1], xv.x, xv.y);
          mma_16816<F16>(acc[nt], o0[2], o1[2], o0[3], o1[3], xv.z, xv.w);
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(empty_bar(s));
    const int u = u_begin + i;
    const int band = cur_band;
    if (++cur_c == a.kc) {
      cur_c = 0;
      ++cur_band;
    }
    if (i + 1 == nunits || cur_c == 0) {
      const int64_t first_u = static_cast<int64_t>(band) * a.kc;
      if (piece0 == first_u && u == first_u + a.kc - 1) {
        // the whole band ran here: finish it now
        if (!waited) {
          grid_dep_wait();  // X A of this call is ready
          waited = true;
        }
        epilogue_lean(band);
      } else {
        // a piece of a band shared with other CTAs: park it; the CTA whose
        // piece completes the band sums them all (after the stream)
        const int which = piece0 == first_u ? 1 : 0;
        float4 *dst = slot_ptr(blockIdx.x, which);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) __stcg(dst + nt * 32, make_float4(acc[nt][0], acc[nt][1], acc[nt][2], acc[nt][3]));
        (which ? last_band : first_band) = band;
      }
      piece0 = u + 1;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[nt][e] = 0.0f;
    }
    return true;
  };

  // constants of the next two units in registers: one unit's are in
  // flight while another is decoded
  Consts ca, cb, cc;
  if (nunits > 0) load_consts(ca);
  if (nunits > 1) load_consts(cb);
  for (int i = 0; i < nunits; i += 3) {
    if (i + 2 < nunits) load_consts(cc);
    if (!run_unit(i, ca)) break;
    if (i + 1 >= nunits) break;
    if (i + 3 < nunits) load_consts(ca);
    if (!run_unit(i + 1, cb)) break;
    if (i + 2 >= nunits) break;
    if (i + 4 < nunits) load_consts(cb);
    if (!run_unit(i + 2, cc)) break;
  }
  if (warp == 0 && lane == 0) {
    // bounded wait for the copies still in flight (only after an abort)
    for (int j = issued > C::SX ? issued - C::SX : 0; j < issued; ++j) {
      const unsigned long long t0 = globaltimer_ns();
      while (!mbar_try_wait(full_bar(j % C::SX), (j / C::SX) & 1u)) {
        if (globaltimer_ns() - t0 > kWaitTimeoutNs) break;
      }
    }
  }
  grid_dep_launch();
  if (first_band < 0 && last_band < 0) return;
  if (!waited) grid_dep_wait();  // X A ready, band counters zeroed

  // For each parked piece: one release increment of the band's counter once
  // every warp's stores are done; the CTA that brings the count to the
  // band's number of pieces sums the slots of CTAs c0 .. c1 in CTA order
  // (so the result does not depend on which CTA finishes last), applies the
  // low-rank term and stores Y. No CTA waits for another.
  // A bounded group barrier rather than bar.sync: a warp that left after a
  // failed wait (the error word is then set) cannot hold the others for good.
  uint32_t group_phase = 0;
  if (!warp_group_sync(group_bar, group_phase, s_abort)) return;  // every warp's parked pieces are stored
  volatile int *s_last = s_abort + 1;  // [0]: first_band completed here, [1]: last_band
  if (threadIdx.x == 0) {
    __threadfence();
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int band = k == 0 ? first_band : last_band;
      int last = 0;
      if (band >= 0) {
        const int64_t first_u = static_cast<int64_t>(band) * a.kc;
        const int npieces = smallm_cta_of(first_u + a.kc - 1, a.units, grid) - smallm_cta_of(first_u, a.units, grid) + 1;
        const unsigned int prev = atomicAdd(&a.counters[band], 1u);
        last = prev == static_cast<unsigned int>(npieces - 1);
        if (last) a.counters[band] = 0u;  // every piece is in: left zero for the next call
      }
      s_last[k] = last;
    }
  }
  if (!warp_group_sync(group_bar, group_phase, s_abort)) return;
#pragma unroll 1
  for (int k = 0; k < 2; ++k) {
    const int band = k == 0 ? first_band : last_band;
    if (band < 0 || !s_last[k]) continue;
    __threadfence();
    const int64_t first_u = static_cast<int64_t>(band) * a.kc;
    const int c0 = smallm_cta_of(first_u, a.units, grid);
    const int c1 = smallm_cta_of(first_u + a.kc - 1, a.units, grid);
    LoraFrag L0;  // its loads overlap the slot loads below
    if (band_row0(band) < a.N) lora_load(band_row0(band), 0, L0);
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[nt][e] = 0.0f;
    for (int cta = c0; cta <= c1; cta += 4) {
      float4 v[4][NT];
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (cta + j <= c1) {
          const float4 *src = slot_ptr(cta + j, cta + j == c0 ? 1 : 0);
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) v[j][nt] = __ldcg(src + nt * 32);
        }
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (cta + j <= c1) {
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            acc[nt][0] += v[j][nt].x;
            acc[nt][1] += v[j][nt].y;
            acc[nt][2] += v[j][nt].z;
            acc[nt][3] += v[j][nt].w;
          }
        }
    }
    epilogue(band, L0);
  }
}

}  // namespace qlora
