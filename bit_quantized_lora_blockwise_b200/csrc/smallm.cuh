// Few-token forward: Y = X W'^T + B^T-term for M <= 16 tokens, a stream of
// the packed weight with the dequantization done in registers.
//
// The forward of one QLoRA linear (intvml.com "DL0087 QLoRA: 4-bit Quantized
// LoRA", opening paragraph and Figure 1): the base weight is stored as NF4
// codes with double-quantized block constants and is dequantized to bf16
// just before it is multiplied. With a few
// tokens the layer reads 0.516 bytes of packed weight per parameter and does
// 2 M flops with it, so it is bound by HBM. This kernel therefore never
// stages the weight in shared memory: every packed byte is loaded once, by
// the thread that decodes it, straight into the register fragment of a
// warp-level 16x8x16 tensor-core MMA. Only the activations (at most 16
// tokens, L2-resident) go through shared memory, brought in by TMA.
//
// Work split. Rows of W come in bands of 256 (one 16-row tile per compute
// warp), K in chunks of 256 (four quantization blocks). The (band, chunk)
// units, band-major, are divided evenly among a persistent grid (stream-K):
// a CTA runs a contiguous range of units, its 16 warps on the same chunks.
// The pieces of a band computed by different CTAs are parked in fp32 slots
// (at most two per CTA: the band its range starts in and the one it ends
// in); the CTA whose piece completes a band (band counter) sums the slots in
// CTA order, so the result does not depend on timing, and no CTA ever waits
// for another one to be scheduled.
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
  const uint8_t *packed;     // [N, K/2], element 2j in the low nibble
  const uint8_t *q;          // [N K / 64] 8-bit block-constant codes
  const float *scale2;       // [ceil(N K / 64 / 256)] second-level scales
  const __nv_bfloat16 *B;    // [r, N]
  const __nv_bfloat16 *xas;  // [M, r] = bf16((alpha / r) X A)
  __nv_bfloat16 *Y;          // [M, N]
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
  static constexpr int THREADS = WARPS * 32;     // lane 0 of warp 0 also issues the X copies
  static constexpr int XR = 8 * NT;              // token rows per stage
  static constexpr int STAGE = 4 * XR * 128;     // [XR tokens][4 blocks][64 bf16]
  static constexpr int SX = 8;                   // activation stages
  static constexpr int OFF_BAR = SX * STAGE;
  static constexpr int OFF_T8 = OFF_BAR + 2 * SX * 8;
  static constexpr int OFF_MISC = OFF_T8 + 256 * 4;  // abort flag, two completed-band flags
  static constexpr int SMEM_BYTES = OFF_MISC + 16;
  static constexpr int SLOT_FLOATS = WARPS * NT * 32 * 4;
  static_assert(STAGE % 1024 == 0, "stages keep the 1024-byte swizzle alignment");
};

// CTA that owns unit u when `units` units are split evenly over `grid` CTAs
// (CTA i runs [floor(i units / grid), floor((i+1) units / grid))).
__host__ __device__ __forceinline__ int smallm_cta_of(int64_t u, int64_t units, int64_t grid) {
  return static_cast<int>(((u + 1) * grid - 1) / units);
}
__host__ __device__ __forceinline__ int smallm_unit_begin(int64_t cta, int64_t units, int64_t grid) {
  return static_cast<int>(cta * units / grid);
}

template <int NT, bool V8>
__global__ void __launch_bounds__(SmallmCfg<NT>::THREADS, 1) smallm_kernel(const __grid_constant__ SmallmArgs a) {
  using C = SmallmCfg<NT>;
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float *s_t8 = reinterpret_cast<float *>(smem + C::OFF_T8);
  volatile int *s_abort = reinterpret_cast<volatile int *>(smem + C::OFF_MISC);
  auto x_full = [&](int s) { return sbase + C::OFF_BAR + 8u * s; };
  auto x_empty = [&](int s) { return sbase + C::OFF_BAR + 8u * (C::SX + s); };

  const int grid = gridDim.x;
  const int u_begin = smallm_unit_begin(blockIdx.x, a.units, grid);
  const int u_end = smallm_unit_begin(blockIdx.x + 1, a.units, grid);
  const int nunits = u_end - u_begin;

  // X copies (lane 0 of warp 0): unit j goes to stage j % SX once every warp
  // has released unit j - SX. Before unit i is consumed its copy must be
  // issued (waiting for the slowest warp if needed); later ones are issued
  // when their stage is already free. The first SX go out before anything
  // else, ahead of the weight stream.
  int x_issued = 0;
  auto issue_x = [&](int i) {
    while (x_issued < nunits && x_issued < i + C::SX) {
      const int j = x_issued, st = j % C::SX;
      if (j >= C::SX) {
        const uint32_t par = ((j / C::SX) - 1) & 1u;
        if (j == i) {
          if (!mbar_wait_spin(x_empty(st), par, s_abort)) return;
        } else if (!mbar_try_wait(x_empty(st), par)) {
          return;
        }
      }
      const int c = (j + u_begin) % a.kc;
      mbar_arrive_expect_tx(x_full(st), C::STAGE);
      tma_load_3d(sbase + st * C::STAGE, &a.tm_x, x_full(st), 0, c * 4, 0);
      ++x_issued;
    }
  };
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::SX; ++s) {
      mbar_init(x_full(s), 1);
      mbar_init(x_empty(s), C::WARPS);
    }
    *s_abort = 0;
    fence_barrier_init();
    tma_prefetch_desc(&a.tm_x);
    issue_x(0);
  }
  for (int i = threadIdx.x; i < 256; i += blockDim.x) s_t8[i] = a.tabs.t8[i];
  __syncthreads();

  // ------------------------------------------------------ compute warps --
  const int g = lane >> 2, t = lane & 3;
  const uint32_t swz = static_cast<uint32_t>((4 * g + t) & 7);
  const int64_t kb_total = a.K / 64;
  const int64_t row_bytes = a.K / 2;

  // This lane's packed bytes, constant codes and scales for one unit. The
  // loader walks the CTA's units in order (chunk by chunk, band by band),
  // so addresses advance by a fixed step inside a band.
  struct Frag {
    uint32_t w[2][8];
    uint32_t q[2];
    float s[2];
  };
  // L2 prefetch: a second walk over the same units, kPfAhead units ahead of
  // the register loads, so that those loads hit L2 rather than DRAM
  constexpr int kPfAhead = 4;
  int pf_band = u_begin / a.kc, pf_c = u_begin - (u_begin / a.kc) * a.kc, pf_idx = 0;
  const uint8_t *pf_p = nullptr, *pf_q = nullptr;
  bool pf_row_ok = false;
  auto pf_setup = [&]() {
    const int64_t row = static_cast<int64_t>(pf_band) * C::BAND + warp * 16 + g;
    pf_row_ok = row < a.N;
    const int64_t bi = row * kb_total + static_cast<int64_t>(pf_c) * 4 + t;
    pf_p = a.packed + bi * 32;
    pf_q = a.q + bi;
  };
  auto pf_step = [&]() {  // prefetch the walk's unit (rows g and g + 8), then advance
    if (pf_idx >= nunits) return;
    if (pf_row_ok && static_cast<int64_t>(pf_c) * 4 + t < kb_total) {
      prefetch_l2(pf_p);
      prefetch_l2(pf_p + 8 * row_bytes);
      prefetch_l2(pf_q);
      prefetch_l2(pf_q + 8 * kb_total);
    }
    ++pf_idx;
    if (++pf_c == a.kc) {
      pf_c = 0;
      ++pf_band;
      pf_setup();
    } else {
      pf_p += 128;
      pf_q += 4;
    }
  };
  pf_setup();
  for (int k = 0; k < kPfAhead; ++k) pf_step();  // units 0 .. kPfAhead - 1 up front
  int ld_band = u_begin / a.kc, ld_c = u_begin - (u_begin / a.kc) * a.kc;
  const uint8_t *ld_p = nullptr;  // row g of the band, chunk ld_c, block t
  int64_t ld_bi = 0;              // block index of that row and block
  bool ld_row_ok = false;
  auto band_setup = [&]() {
    const int64_t row = static_cast<int64_t>(ld_band) * C::BAND + warp * 16 + g;
    ld_row_ok = row < a.N;
    ld_bi = row * kb_total + static_cast<int64_t>(ld_c) * 4 + t;
    ld_p = a.packed + ld_bi * 32;
  };
  band_setup();
  auto load_next = [&](Frag &f) {
    const bool ok = ld_row_ok && static_cast<int64_t>(ld_c) * 4 + t < kb_total;
    if (ok) {
#pragma unroll
      for (int rr = 0; rr < 2; ++rr) {
        const uint8_t *p = ld_p + rr * 8 * row_bytes;
        if (V8) {
          ld_stream_32B(p, f.w[rr]);
        } else {
          const uint4 lo = ld_stream_16B(p), hi = ld_stream_16B(p + 16);
          f.w[rr][0] = lo.x; f.w[rr][1] = lo.y; f.w[rr][2] = lo.z; f.w[rr][3] = lo.w;
          f.w[rr][4] = hi.x; f.w[rr][5] = hi.y; f.w[rr][6] = hi.z; f.w[rr][7] = hi.w;
        }
        const int64_t bi = ld_bi + rr * 8 * kb_total;
        f.q[rr] = __ldg(a.q + bi);
        f.s[rr] = __ldg(a.scale2 + (bi >> 8));
      }
    } else {
#pragma unroll
      for (int rr = 0; rr < 2; ++rr) {
#pragma unroll
        for (int j = 0; j < 8; ++j) f.w[rr][j] = 0u;
        f.q[rr] = 0u;
        f.s[rr] = 0.0f;  // c' = 0: the block contributes zeros
      }
    }
    if (++ld_c == a.kc) {
      ld_c = 0;
      ++ld_band;
      band_setup();
    } else {
      ld_p += 128;
      ld_bi += 4;
    }
    pf_step();
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
        mma_16816_bf16(acc[nt], L.af[q][0], L.af[q][1], L.af[q][2], L.af[q][3], L.bf[q][nt][0], L.bf[q][nt][1]);
  };
  auto band_row0 = [&](int band) { return static_cast<int64_t>(band) * C::BAND + warp * 16; };
  auto store_y = [&](int64_t n0) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int m = 8 * nt + 2 * t + (e & 1);
        const int64_t n = n0 + g + 8 * (e >> 1);
        if (m < a.M) a.Y[static_cast<int64_t>(m) * a.N + n] = __float2bfloat16_rn(acc[nt][e]);
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
        mma_16816_bf16(acc[nt], a0, a1, a2, a3, b0, b1);
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

  const uint32_t swz16 = swz << 4;
  const uint32_t xrow = sbase + static_cast<uint32_t>((4 * g + t) * 128);
  int cur_band = ld_band, cur_c = ld_c, piece0 = u_begin;
  // Decode one unit's codes into MMA fragments and accumulate; then
  // release its activation stage and close the piece if a band ends.
  auto run_unit = [&](int i, const Frag &f) -> bool {
    const float cp0 = __fmul_rn(s_t8[f.q[0]], f.s[0]);
    const float cp1 = __fmul_rn(s_t8[f.q[1]], f.s[1]);
    const Nf4Planes P0 = make_planes(a.tabs.nf4, cp0);
    const Nf4Planes P1 = make_planes(a.tabs.nf4, cp1);
    const int s = i % C::SX;
    if (warp == 0 && lane == 0) issue_x(i);
    __syncwarp();
    if (!__all_sync(0xFFFFFFFFu, mbar_wait_spin(x_full(s), (i / C::SX) & 1u, s_abort))) return false;
    const uint32_t xs = xrow + s * C::STAGE;
    const bool rows_here = static_cast<int64_t>(cur_band) * C::BAND + warp * 16 < a.N;
#pragma unroll
    for (int uu = 0; uu < (rows_here ? 8 : 0); ++uu) {
      uint32_t o0[4], o1[4];
      nf4_lookup8(P0, f.w[0][uu], o0);
      nf4_lookup8(P1, f.w[1][uu], o1);
      const uint32_t xa = xs | ((static_cast<uint32_t>(uu) << 4) ^ swz16);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const uint4 xv = lds_16B(xa + nt * (8 * 4 * 128));
        mma_16816_bf16(acc[nt], o0[0], o1[0], o0[1], o1[1], xv.x, xv.y);
        mma_16816_bf16(acc[nt], o0[2], o1[2], o0[3], o1[3], xv.z, xv.w);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(x_empty(s));
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

  // two register buffers: the next unit's loads are in flight while one
  // unit is decoded
  Frag fa, fb;
  if (nunits > 0) load_next(fa);
  for (int i = 0; i < nunits; i += 2) {
    if (i + 1 < nunits) load_next(fb);
    if (!run_unit(i, fa)) break;
    if (i + 1 >= nunits) break;
    if (i + 2 < nunits) load_next(fa);
    if (!run_unit(i + 1, fb)) break;
  }
  if (warp == 0 && lane == 0) {
    // bounded wait for X copies still in flight (only after an abort)
    for (int j = x_issued > C::SX ? x_issued - C::SX : 0; j < x_issued; ++j) {
      const unsigned long long t0 = globaltimer_ns();
      while (!mbar_try_wait(x_full(j % C::SX), (j / C::SX) & 1u)) {
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
  named_bar_sync(1, C::WARPS * 32);  // every warp's parked pieces are stored
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
  named_bar_sync(1, C::WARPS * 32);
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
