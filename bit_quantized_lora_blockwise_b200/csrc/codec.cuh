// NF4 codec kernels: blockwise absmax + nearest-level encode + nibble pack,
// double quantization of the absmax constants, and dequantization to bf16.
//
// Method (QLoRA pages): intvml.com "DL0087 QLoRA: 4-bit Quantized LoRA",
// components (1)-(3) and the formulation's symbol list; promptingindex.com
// "QLoRA: Finetuning 65B Models on a Single GPU", sections "4-bit
// NormalFloat" and "Double Quantization and Paged Optimizers".
//
// Quantize and dequant are HBM-bound streaming kernels: wide vector loads
// (one lane takes 16 consecutive weights to quantize, or a whole 64-block to
// dequantize), warp shuffles for the per-block reduction, grid-stride loops
// over a grid sized to the SM count. Double quantization has far fewer
// bytes and is bound by latency: one warp per group of 256 constants.
#pragma once

#include "ptx.cuh"

namespace qlora {

struct CodecTables {
  float nf4[16];
  float t8[256];
};

// ------------------------------------------------------------------------
// NF4 code of x: the number of fp32 midpoints m_i = (L_i + L_{i+1}) * 0.5
// strictly below x, by a 4-step binary search over the 15 sorted midpoints
// (mid[] in shared memory, mid7 in a register).
__device__ __forceinline__ uint32_t nf4_code(float x, const float *mid, float mid7) {
  uint32_t c = (x > mid7) ? 8u : 0u;
  c += (x > mid[c + 3]) ? 4u : 0u;
  c += (x > mid[c + 1]) ? 2u : 0u;
  c += (x > mid[c]) ? 1u : 0u;
  return c;
}

// Correctly rounded x = w / c from the correctly rounded reciprocal
// r = RN(1/c): q0 = RN(w r), residual e = w - q0 c (exact with one FMA),
// x = RN(q0 + e r). Markstein's theorem (P. Markstein, "Computation of
// elementary functions on the IBM RISC System/6000 processor", IBM J. Res.
// Dev. 34(1), 1990) gives x = RN(w / c) when r is within half an ulp of 1/c
// and q0 within one ulp of w / c, barring underflow. The caller routes
// blocks whose c lies outside [2^-125, 2^125] (1/c near overflow or
// subnormal) through the IEEE divide; a quotient that underflows is far
// below every NF4 midpoint, so its rounding cannot change the code.
__device__ __forceinline__ float div_by_recip(float w, float c, float r) {
  const float q0 = __fmul_rn(w, r);
  const float e = __fmaf_rn(-q0, c, w);
  return __fmaf_rn(e, r, q0);
}

// Bucketed encode. y = RN(128 x + 128 + 1.5 * 2^23) rounds 128 x + 128 to an
// integer t in [0, 256] (|x| <= 1; the ulp at that magnitude is 1) and is
// monotone in x. Bucket j = t / 8 (width 1/16) is an interval of x values;
// as the magic's low 22 bits are zero, bits(y) & 0x1F8 = 8 j is directly the
// byte offset of the bucket's 8-byte entry, and a 64-entry table keeps any
// input (even a non-finite one) in range. The host builds, for each bucket,
// the code of its first x (cand) and the one midpoint that falls strictly
// inside it (thr; 2.0 when none), after checking that no bucket holds two;
// then code(x) = cand[j] + (x > thr[j]) exactly. Tables whose midpoints are
// closer than a bucket width (1/16) use the binary search instead.
struct BucketTable {
  float thr[33];
  unsigned int cand[33];
};
constexpr float kBucketMagic = 12582912.0f;  // 1.5 * 2^23

__device__ __forceinline__ float2 bucket_entry(const float2 *bk, float y) {
  return *reinterpret_cast<const float2 *>(reinterpret_cast<const char *>(bk) + (__float_as_uint(y) & 0x1F8u));
}

// 0xFFFFFFFF when a > b, else 0 (false for NaN)
__device__ __forceinline__ uint32_t set_gt_mask(float a, float b) {
  uint32_t r;
  asm("set.gt.u32.f32 %0, %1, %2;" : "=r"(r) : "f"(a), "f"(b));
  return r;
}

__device__ __forceinline__ uint32_t nf4_code_bucket(float x, const float2 *bk) {
  const float2 e = bucket_entry(bk, __fmaf_rn(x, 128.0f, 128.0f + kBucketMagic));
  return __float_as_uint(e.y) + (x > e.x ? 1u : 0u);
}

// Encode of one 64-block slice: 8 weights (one 16-byte word) -> 8 nibbles.
// The bucketed path runs the division and the bucket map on fp32 pairs
// (f32x2 FMA/MUL: two IEEE round-to-nearest lanes per instruction) and packs
// nibbles with one multiply-add each.
template <bool BUCKET>
__device__ __forceinline__ uint32_t encode8(const float (&f)[8], float c, const float *s_mid, float mid7,
                                            const float2 *s_bk) {
  if (BUCKET && c >= 0x1p-125f && c <= 0x1p125f) {
    const float r = __frcp_rn(c);
    const unsigned long long R = f2_pack(r, r), NC = f2_pack(-c, -c);
    const unsigned long long S128 = f2_pack(128.0f, 128.0f);
    const unsigned long long OFF = f2_pack(128.0f + kBucketMagic, 128.0f + kBucketMagic);
    uint32_t word = 0;
#pragma unroll
    for (int i = 3; i >= 0; --i) {  // pairs (6,7), (4,5), ... so the word fills from the top nibble
      const unsigned long long W = f2_pack(f[2 * i], f[2 * i + 1]);
      const unsigned long long Q0 = f2_mul(W, R);       // RN(w r)
      const unsigned long long E = f2_fma(Q0, NC, W);   // w - q0 c, exact
      const unsigned long long X = f2_fma(E, R, Q0);    // RN(q0 + e r) = RN(w / c)
      const unsigned long long Y = f2_fma(X, S128, OFF);  // bucket map
      float x0, x1, y0, y1;
      f2_unpack(X, x0, x1);
      f2_unpack(Y, y0, y1);
      const float2 e1 = bucket_entry(s_bk, y1), e0 = bucket_entry(s_bk, y0);
      // code = cand + (x > thr): the compare gives an all-ones mask, subtracted
      word = word * 16u + __float_as_uint(e1.y) - set_gt_mask(x1, e1.x);
      word = word * 16u + __float_as_uint(e0.y) - set_gt_mask(x0, e0.x);
    }
    return word;
  }
  auto code = [&](float x) -> uint32_t {
    return BUCKET ? nf4_code_bucket(x, s_bk) : nf4_code(x, s_mid, mid7);
  };
  uint32_t word = 0;
  if (c == 0.0f) {
    word = code(0.0f) * 0x11111111u;
  } else if (c >= 0x1p-125f && c <= 0x1p125f) {
    const float r = __frcp_rn(c);
#pragma unroll
    for (int i = 0; i < 8; ++i) word |= code(div_by_recip(f[i], c, r)) << (4 * i);
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) word |= code(__fdiv_rn(f[i], c)) << (4 * i);
  }
  return word;
}

// One 64-weight block per 4 lanes; each lane encodes 16 consecutive weights
// (one 32-byte load, or two 16-byte loads when W is only 16-byte aligned)
// into two 32-bit words of 8 nibbles. A warp takes 16 blocks per iteration
// (two independent loads per lane in flight), and the next iteration's loads
// are issued before this one is encoded.
template <bool BUCKET, bool V8>
__global__ void __launch_bounds__(256) quantize_nf4_kernel(const uint4 *__restrict__ W,
                                                           int64_t nblocks,
                                                           uint32_t *__restrict__ packed,
                                                           float *__restrict__ absmax,
                                                           const CodecTables tabs, const BucketTable bt) {
  __shared__ float s_mid[16];
  // 33 buckets, padded to 64 so that every offset bits(y) & 0x1F8 is in range;
  // a NaN quotient (NaN weight, or inf / inf) lands in a padding entry and
  // gets code 0, as no midpoint lies strictly below NaN
  __shared__ float2 s_bk[64];
  if (threadIdx.x < 15)
    s_mid[threadIdx.x] = __fmul_rn(__fadd_rn(tabs.nf4[threadIdx.x], tabs.nf4[threadIdx.x + 1]), 0.5f);
  if (threadIdx.x < 64)
    s_bk[threadIdx.x] = threadIdx.x < 33 ? make_float2(bt.thr[threadIdx.x], __uint_as_float(bt.cand[threadIdx.x]))
                                         : make_float2(2.0f, __uint_as_float(0u));
  __syncthreads();
  grid_dep_wait();
  grid_dep_launch();
  const float mid7 = s_mid[7];
  const uint32_t lane = threadIdx.x & 31u;
  const int64_t nunits = nblocks * 4;  // 32-byte units of 16 weights
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x * 2;
  // The loop runs per warp (base is warp-uniform) so the shuffles below
  // always see all 32 lanes; lanes past the end compute on zeros.
  int64_t base = (static_cast<int64_t>(blockIdx.x) * blockDim.x + (threadIdx.x & ~31u)) * 2;
  uint32_t vn[2][8];
  auto load = [&](int64_t b) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int64_t t = b + 32 * h + lane;
      if (t < nunits) {
        if (V8) {
          ld_stream_32B(W + 2 * t, vn[h]);
        } else {
          const uint4 lo = __ldg(W + 2 * t), hi = __ldg(W + 2 * t + 1);
          vn[h][0] = lo.x; vn[h][1] = lo.y; vn[h][2] = lo.z; vn[h][3] = lo.w;
          vn[h][4] = hi.x; vn[h][5] = hi.y; vn[h][6] = hi.z; vn[h][7] = hi.w;
        }
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) vn[h][i] = 0u;
      }
    }
  };
  if (base < nunits) load(base);
  for (; base < nunits; base += stride) {
    uint32_t v[2][8];
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int i = 0; i < 8; ++i) v[h][i] = vn[h][i];
    if (base + stride < nunits) load(base + stride);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int64_t t = base + 32 * h + lane;
      float f0[8], f1[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        f0[2 * i] = __uint_as_float(v[h][i] << 16);
        f0[2 * i + 1] = __uint_as_float(v[h][i] & 0xFFFF0000u);
        f1[2 * i] = __uint_as_float(v[h][4 + i] << 16);
        f1[2 * i + 1] = __uint_as_float(v[h][4 + i] & 0xFFFF0000u);
      }
      float m = 0.0f;
#pragma unroll
      for (int i = 0; i < 8; ++i) m = fmaxf(m, fmaxf(fabsf(f0[i]), fabsf(f1[i])));
      // each 4-lane group (one 64-block) reduces independently
      m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
      m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
      const uint32_t w0 = encode8<BUCKET>(f0, m, s_mid, mid7, s_bk);
      const uint32_t w1 = encode8<BUCKET>(f1, m, s_mid, mid7, s_bk);
      if (t < nunits) {
        *reinterpret_cast<uint2 *>(packed + 2 * t) = make_uint2(w0, w1);
        if ((lane & 3u) == 0) absmax[t >> 2] = m;
      }
    }
  }
}

// ------------------------------------------------------------------------
// Double quantization: one warp per group of 256 constants, 8 per lane.
// S = group max; q = number of fp32 midpoints of t8 strictly below
// x = RN(c / S); a group of zeros gives x = 0.
//
// Bucketed search. With every midpoint m in [2^-100, 1] and no two closer
// than 1/256, y = RN(256 x + 1.5 * 2^23) gives j = bits(y) - bits(1.5 * 2^23)
// = RNE(256 x) in [0, 256] for x in [0, 1]: a monotone map onto 257 buckets
// of width 1/256 with at most one midpoint strictly inside each. The host
// fills cand[j] (midpoints below every x of bucket j) and thr[j] (the one
// inside, 2.0 when none) and checks those conditions; then
// q = cand[j] + (x > thr[j]). Any other j (x < -1/512 or NaN: no midpoint
// lies strictly below such an x) is clamped to entry 257, which gives 0.
// Tables that fail the check use an 8-step binary search over the 255
// midpoints instead.
struct DqBucketTable {
  float thr[258];
  unsigned int cand[258];
};

template <bool BUCKET>
__global__ void __launch_bounds__(256) double_quant_kernel(const float *__restrict__ absmax,
                                                           int64_t nb, uint8_t *__restrict__ q,
                                                           float *__restrict__ scale2,
                                                           const CodecTables tabs, const DqBucketTable bt) {
  __shared__ float s_mid[BUCKET ? 1 : 256];
  __shared__ float2 s_bk[BUCKET ? 258 : 1];
  if constexpr (BUCKET) {
    for (int i = threadIdx.x; i < 258; i += blockDim.x)
      s_bk[i] = make_float2(bt.thr[i], __uint_as_float(bt.cand[i]));
  } else {
    if (threadIdx.x < 255)
      s_mid[threadIdx.x] = __fmul_rn(__fadd_rn(tabs.t8[threadIdx.x], tabs.t8[threadIdx.x + 1]), 0.5f);
  }
  __syncthreads();
  grid_dep_wait();
  grid_dep_launch();
  const int lane = threadIdx.x & 31;
  const int64_t ng = (nb + 255) / 256;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  // this lane's 8 constants of group g (zeros past the end)
  auto load = [&](int64_t g, float (&c)[8]) {
    const int64_t base = g * 256 + lane * 8;
    if (base + 8 <= nb) {
      const float4 a = __ldg(reinterpret_cast<const float4 *>(absmax + base));
      const float4 b = __ldg(reinterpret_cast<const float4 *>(absmax + base + 4));
      c[0] = a.x; c[1] = a.y; c[2] = a.z; c[3] = a.w;
      c[4] = b.x; c[5] = b.y; c[6] = b.z; c[7] = b.w;
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) c[i] = (base + i < nb) ? absmax[base + i] : 0.0f;
    }
  };
  int64_t g = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  float cn[8];
  if (g < ng) load(g, cn);
  for (; g < ng; g += warps) {
    float c[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) c[i] = cn[i];
    if (g + warps < ng) load(g + warps, cn);  // the next group's loads go out first
    float s = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) s = fmaxf(s, c[i]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s = fmaxf(s, __shfl_xor_sync(0xFFFFFFFFu, s, o));
    uint32_t codes[8];
    if constexpr (BUCKET) {
      // RN(c / S) through the correctly rounded reciprocal (Markstein, as in
      // encode8) when S is well inside the normal range, else the IEEE divide
      const bool fast = s >= 0x1p-125f && s <= 0x1p125f;
      const float r = fast ? __frcp_rn(s) : 0.0f;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float x = (s == 0.0f) ? 0.0f : (fast ? div_by_recip(c[i], s, r) : __fdiv_rn(c[i], s));
        const float y = __fmaf_rn(x, 256.0f, kBucketMagic);
        const uint32_t j = min(__float_as_uint(y) - __float_as_uint(kBucketMagic), 257u);
        const float2 e = s_bk[j];
        codes[i] = __float_as_uint(e.y) + (x > e.x ? 1u : 0u);
      }
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float x = (s == 0.0f) ? 0.0f : __fdiv_rn(c[i], s);
        uint32_t k = 0;
#pragma unroll
        for (uint32_t step = 128; step > 0; step >>= 1)
          if (x > s_mid[k + step - 1]) k += step;
        codes[i] = k;
      }
    }
    const int64_t base = g * 256 + lane * 8;
    if (base + 8 <= nb) {
      uint2 packed8;
      packed8.x = codes[0] | (codes[1] << 8) | (codes[2] << 16) | (codes[3] << 24);
      packed8.y = codes[4] | (codes[5] << 8) | (codes[6] << 16) | (codes[7] << 24);
      *reinterpret_cast<uint2 *>(q + base) = packed8;
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if (base + i < nb) q[base + i] = static_cast<uint8_t>(codes[i]);
    }
    if (lane == 0) scale2[g] = s;
  }
}

// ------------------------------------------------------------------------
// Quantize fused with the double quantization: one CTA owns whole groups of
// 256 blocks (16384 weights, a second-level group), so the block constants
// never leave the chip. Per group: the 256 threads load 4 units of 16
// weights each (the next group's loads are issued before this one is
// encoded), find every block's absmax across its 4 lanes, encode and store
// the NF4 codes exactly as quantize_nf4_kernel does, and park the absmax in
// shared memory; then thread i encodes constant i of the group as
// double_quant_kernel does (S = the group's max, q = the 8-bit code of
// RN(c / S)) and the CTA writes q and S (and the fp32 absmax only when the
// caller asks for it). Bytes: 2 read + 0.5 + 1/64 + 4/16384 written per
// weight.
template <bool BUCKET>
__device__ __forceinline__ uint32_t dq_code(float c, float s, float r, bool fast, const float2 *s_bk,
                                            const float *s_mid) {
  if constexpr (BUCKET) {
    const float x = (s == 0.0f) ? 0.0f : (fast ? div_by_recip(c, s, r) : __fdiv_rn(c, s));
    const float y = __fmaf_rn(x, 256.0f, kBucketMagic);
    const uint32_t j = min(__float_as_uint(y) - __float_as_uint(kBucketMagic), 257u);
    const float2 e = s_bk[j];
    return __float_as_uint(e.y) + (x > e.x ? 1u : 0u);
  } else {
    const float x = (s == 0.0f) ? 0.0f : __fdiv_rn(c, s);
    uint32_t k = 0;
#pragma unroll
    for (uint32_t step = 128; step > 0; step >>= 1)
      if (x > s_mid[k + step - 1]) k += step;
    return k;
  }
}

template <bool BUCKET, bool V8, bool DQBUCKET, int QT = 256>
__global__ void __launch_bounds__(QT) quantize_dq_kernel(const uint4 *__restrict__ W, int64_t nblocks,
                                                          uint32_t *__restrict__ packed, uint8_t *__restrict__ q,
                                                          float *__restrict__ scale2, float *__restrict__ absmax,
                                                          const CodecTables tabs, const BucketTable bt,
                                                          const DqBucketTable dbt) {
  __shared__ float s_mid[16];
  __shared__ float2 s_bk[64];
  __shared__ float s_mid8[DQBUCKET ? 1 : 256];
  __shared__ float2 s_bk8[DQBUCKET ? 258 : 1];
  __shared__ float s_c[2][256];  // the group's constants (two buffers: no barrier between groups)
  __shared__ float s_wmax[2][8];
  static_assert(QT == 256 || QT == 512 || QT == 1024, "threads per CTA");
  const int tid = threadIdx.x;
  if (tid < 15) s_mid[tid] = __fmul_rn(__fadd_rn(tabs.nf4[tid], tabs.nf4[tid + 1]), 0.5f);
  if (tid < 64)
    s_bk[tid] = tid < 33 ? make_float2(bt.thr[tid], __uint_as_float(bt.cand[tid])) : make_float2(2.0f, 0.0f);
  if constexpr (DQBUCKET) {
    for (int i = tid; i < 258; i += blockDim.x) s_bk8[i] = make_float2(dbt.thr[i], __uint_as_float(dbt.cand[i]));
  } else {
    if (tid < 255) s_mid8[tid] = __fmul_rn(__fadd_rn(tabs.t8[tid], tabs.t8[tid + 1]), 0.5f);
  }
  __syncthreads();
  grid_dep_wait();
  grid_dep_launch();
  const float mid7 = s_mid[7];
  const int64_t nunits = nblocks * 4;     // 32-byte units of 16 weights
  const int64_t ng = (nblocks + 255) / 256;
  constexpr int U = 1024 / QT;             // units per thread per group: QT threads x U = 1024 units = 256 blocks
  uint32_t vn[U][8];
  auto load = [&](int64_t g) {
#pragma unroll
    for (int h = 0; h < U; ++h) {
      const int64_t t = g * 1024 + h * QT + tid;
      if (t < nunits) {
        if (V8) {
          ld_stream_32B(W + 2 * t, vn[h]);
        } else {
          const uint4 lo = __ldg(W + 2 * t), hi = __ldg(W + 2 * t + 1);
          vn[h][0] = lo.x; vn[h][1] = lo.y; vn[h][2] = lo.z; vn[h][3] = lo.w;
          vn[h][4] = hi.x; vn[h][5] = hi.y; vn[h][6] = hi.z; vn[h][7] = hi.w;
        }
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) vn[h][i] = 0u;
      }
    }
  };
  int64_t g = blockIdx.x;
  if (g < ng) load(g);
  for (int buf = 0; g < ng; g += gridDim.x, buf ^= 1) {
    uint32_t v[U][8];
#pragma unroll
    for (int h = 0; h < U; ++h)
#pragma unroll
      for (int i = 0; i < 8; ++i) v[h][i] = vn[h][i];
    if (g + gridDim.x < ng) load(g + gridDim.x);
#pragma unroll
    for (int h = 0; h < U; ++h) {
      const int64_t t = g * 1024 + h * QT + tid;
      float f0[8], f1[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        f0[2 * i] = __uint_as_float(v[h][i] << 16);
        f0[2 * i + 1] = __uint_as_float(v[h][i] & 0xFFFF0000u);
        f1[2 * i] = __uint_as_float(v[h][4 + i] << 16);
        f1[2 * i + 1] = __uint_as_float(v[h][4 + i] & 0xFFFF0000u);
      }
      float m = 0.0f;
#pragma unroll
      for (int i = 0; i < 8; ++i) m = fmaxf(m, fmaxf(fabsf(f0[i]), fabsf(f1[i])));
      m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
      m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
      const uint32_t w0 = encode8<BUCKET>(f0, m, s_mid, mid7, s_bk);
      const uint32_t w1 = encode8<BUCKET>(f1, m, s_mid, mid7, s_bk);
      if (t < nunits) *reinterpret_cast<uint2 *>(packed + 2 * t) = make_uint2(w0, w1);
      // block (h * 256 + tid) / 4 of the group; zeros past the last block
      if ((tid & 3) == 0) s_c[buf][(h * QT + tid) >> 2] = t < nunits ? m : 0.0f;
    }
    __syncthreads();
    // second level: constant tid of the group (the first 256 threads)
    const int64_t b = g * 256 + tid;
    const float c = tid < 256 ? s_c[buf][tid] : 0.0f;
    float s = c;
    if (tid < 256) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) s = fmaxf(s, __shfl_xor_sync(0xFFFFFFFFu, s, o));
      if ((tid & 31) == 0) s_wmax[buf][tid >> 5] = s;
    }
    __syncthreads();
    if (tid < 256) {
      s = s_wmax[buf][0];
#pragma unroll
      for (int w = 1; w < 8; ++w) s = fmaxf(s, s_wmax[buf][w]);
      const bool fast = s >= 0x1p-125f && s <= 0x1p125f;
      const float r = (DQBUCKET && fast) ? __frcp_rn(s) : 0.0f;
      const uint32_t code = dq_code<DQBUCKET>(c, s, r, fast, s_bk8, s_mid8);
      if (b < nblocks) {
        q[b] = static_cast<uint8_t>(code);
        if (absmax != nullptr) absmax[b] = c;
      }
      if (tid == 0) scale2[g] = s;
    }
  }
}

// ------------------------------------------------------------------------
// NF4 decode of one block: the 16 products bf16(L_i * c') are formed once
// (fp32 multiply, RNE to bf16) and split into four 8-byte planes (low and
// high bytes of entries 0-7 and 8-15); each 4-bit code then picks its two
// bytes with byte permutes, with no memory lookups.
struct Nf4Planes {
  uint32_t alo0, alo1, ahi0, ahi1, blo0, blo1, bhi0, bhi1;
};

__device__ __forceinline__ Nf4Planes make_planes(const float (&L)[16], float cp, bool f16 = false) {
  uint32_t t[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) t[j] = pack_16x2(__fmul_rn(L[2 * j], cp), __fmul_rn(L[2 * j + 1], cp), f16);
  Nf4Planes p;
  p.alo0 = prmt(t[0], t[1], 0x6420u);
  p.alo1 = prmt(t[2], t[3], 0x6420u);
  p.ahi0 = prmt(t[0], t[1], 0x7531u);
  p.ahi1 = prmt(t[2], t[3], 0x7531u);
  p.blo0 = prmt(t[4], t[5], 0x6420u);
  p.blo1 = prmt(t[6], t[7], 0x6420u);
  p.bhi0 = prmt(t[4], t[5], 0x7531u);
  p.bhi1 = prmt(t[6], t[7], 0x7531u);
  return p;
}

// 8 codes (nibble i of w = element i) -> 8 bf16 in out[0..3]
// (out[k] = element 2k in the low half, 2k+1 in the high half).
__device__ __forceinline__ void nf4_lookup8(const Nf4Planes &P, uint32_t w, uint32_t (&out)[4]) {
  const uint32_t m = w & 0x77777777u;                       // code & 7 of every nibble
  const uint32_t s = ((w >> 1) & 0x44444444u) | 0x32103210u;  // byte k or k+4 by code bit 3
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const uint32_t mh = h ? (m >> 16) : m;
    const uint32_t sh = h ? (s >> 16) : s;
    const uint32_t la = prmt(P.alo0, P.alo1, mh);
    const uint32_t lb = prmt(P.blo0, P.blo1, mh);
    const uint32_t ha = prmt(P.ahi0, P.ahi1, mh);
    const uint32_t hb = prmt(P.bhi0, P.bhi1, mh);
    const uint32_t lo = prmt(la, lb, sh);
    const uint32_t hi = prmt(ha, hb, sh);
    out[2 * h] = prmt(lo, hi, 0x5140u);
    out[2 * h + 1] = prmt(lo, hi, 0x7362u);
  }
}

// Standalone dequantization to bf16, or to fp16 when f16 is set (the pages'
// compute types, systemoverflow.com "QLoRA ... at Extreme Scale": 16-bit
// float or bfloat16): one lane per 64-block (its 16-bit table built once),
// 32 consecutive blocks per warp. Each lane writes its 128 output
// bytes into a padded shared-memory row, and the warp then stores the 4 KB
// with fully coalesced 16-byte stores.
__global__ void __launch_bounds__(256) dequant_kernel(const uint4 *__restrict__ packed,
                                                      const uint8_t *__restrict__ q,
                                                      const float *__restrict__ scale2,
                                                      int64_t nblocks, uint4 *__restrict__ out,
                                                      const CodecTables tabs, int f16) {
  __shared__ float s_t8[256];
  __shared__ uint4 s_stage[8][32 * 9];  // per warp: 32 rows of 128 B, padded to 144 B
  s_t8[threadIdx.x] = tabs.t8[threadIdx.x];
  __syncthreads();
  grid_dep_wait();
  grid_dep_launch();
  float L[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) L[i] = tabs.nf4[i];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  uint4 *stage = s_stage[wid];
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * 8;
  // this lane's block of the next iteration is loaded before the current one
  // is decoded
  uint4 n0 = make_uint4(0u, 0u, 0u, 0u), n1 = n0;
  uint32_t nq = 0u;
  float ns = 0.0f;
  auto load = [&](int64_t b) {
    if (b < nblocks) {
      n0 = __ldg(&packed[2 * b]);
      n1 = __ldg(&packed[2 * b + 1]);
      nq = __ldg(&q[b]);
      ns = __ldg(&scale2[b >> 8]);
    } else {
      n0 = n1 = make_uint4(0u, 0u, 0u, 0u);
      nq = 0u;
      ns = 0.0f;
    }
  };
  int64_t b0 = (static_cast<int64_t>(blockIdx.x) * 8 + wid) * 32;
  if (b0 < nblocks) load(b0 + lane);
  for (; b0 < nblocks; b0 += nwarps * 32) {
    const uint4 w0 = n0, w1 = n1;
    const float cp = __fmul_rn(s_t8[nq], ns);
    if (b0 + nwarps * 32 < nblocks) load(b0 + nwarps * 32 + lane);
    const Nf4Planes P = make_planes(L, cp, f16 != 0);
    const uint32_t words[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      uint32_t o[4];
      nf4_lookup8(P, words[c], o);
      stage[lane * 9 + c] = make_uint4(o[0], o[1], o[2], o[3]);
    }
    __syncwarp();
    const int64_t nvalid = nblocks - b0 < 32 ? nblocks - b0 : 32;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int idx = i * 32 + lane;  // 16-byte chunk of the warp's 4 KB
      const int row = idx >> 3, ch = idx & 7;
      if (row < nvalid) out[b0 * 8 + idx] = stage[row * 9 + ch];
    }
    __syncwarp();
  }
}


}  // namespace qlora
