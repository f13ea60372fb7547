// Paged AdamW for the adapters (intvml.com "DL0087 QLoRA: 4-bit Quantized
// LoRA", component (5) "Paged Optimizers"; promptingindex.com "QLoRA:
// Finetuning 65B Models on a Single GPU", section "Double Quantization and
// Paged Optimizers"): the optimizer state lives in unified (managed) memory
// so that, when device memory runs short (the spikes of gradient
// checkpointing on long sequences), it can be paged out to host RAM and
// back instead of failing the step.
//
// The update is AdamW with decoupled weight decay (I. Loshchilov and
// F. Hutter, "Decoupled Weight Decay Regularization", ICLR 2019,
// Algorithm 2), in fp32 on an fp32 master copy of the 16-bit adapter
// parameters; the 16-bit parameters are the master rounded to nearest even:
//   p <- p (1 - lr wd)
//   m <- b1 m + (1 - b1) g
//   v <- b2 v + (1 - b2) g^2
//   p <- p - (lr / (1 - b1^t)) m / (sqrt(v / (1 - b2^t)) + eps)
// One pass over HBM (or over host memory, when the state is paged out):
// 2 bytes of gradient in, 12 bytes of state read and written, 2 bytes of
// parameter out per element. The grid strides over segments (one adapter
// tensor each) of up to kAdamwMaxSegs tensors per launch.
#pragma once

#include "ptx.cuh"

namespace qlora {

constexpr int kAdamwMaxSegs = 32;

struct AdamwSegs {
  void *param[kAdamwMaxSegs];        // 16-bit parameters [count]
  const void *grad[kAdamwMaxSegs];   // 16-bit gradients [count]
  int64_t offset[kAdamwMaxSegs + 1]; // element offsets of the segments in the state
  int nseg;
};

struct AdamwHyper {
  float lr, b1, b2, eps, wd;
  float bc1, bc2;  // 1 - b1^t and 1 - b2^t (from the host, in double then rounded)
  int f16;         // 16-bit type of param and grad (else bf16)
};

__device__ __forceinline__ float from_16(uint16_t h, bool f16) {
  return f16 ? __half2float(__ushort_as_half(h)) : __bfloat162float(__ushort_as_bfloat16(h));
}

// master, m, v: fp32 [total] each (managed memory). Element i of the state
// belongs to the segment whose [offset[s], offset[s+1]) holds it.
__global__ void __launch_bounds__(256) adamw_kernel(const AdamwSegs segs, float *__restrict__ master,
                                                    float *__restrict__ m, float *__restrict__ v,
                                                    const AdamwHyper h) {
  grid_dep_wait();  // the gradients come from the kernels before
  grid_dep_launch();
  const bool f16 = h.f16 != 0;
  const int64_t total = segs.offset[segs.nseg];
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const float decay = 1.0f - h.lr * h.wd;
  const float step = h.lr / h.bc1;
  int s = 0;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total; i += stride) {
    while (i >= segs.offset[s + 1]) ++s;  // i only grows: the segment index only moves forward
    const int64_t j = i - segs.offset[s];
    const float g = from_16(static_cast<const uint16_t *>(segs.grad[s])[j], f16);
    float p = master[i] * decay;
    const float mi = h.b1 * m[i] + (1.0f - h.b1) * g;
    const float vi = h.b2 * v[i] + (1.0f - h.b2) * (g * g);
    p -= step * mi / (sqrtf(vi / h.bc2) + h.eps);
    master[i] = p;
    m[i] = mi;
    v[i] = vi;
    static_cast<uint16_t *>(segs.param[s])[j] = to_16(p, f16);
  }
}

// master <- the 16-bit parameters, m = v = 0 (the optimizer's start).
__global__ void __launch_bounds__(256) adamw_init_kernel(const AdamwSegs segs, float *__restrict__ master,
                                                         float *__restrict__ m, float *__restrict__ v, int f16) {
  grid_dep_wait();
  grid_dep_launch();
  const int64_t total = segs.offset[segs.nseg];
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  int s = 0;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total; i += stride) {
    while (i >= segs.offset[s + 1]) ++s;
    const int64_t j = i - segs.offset[s];
    master[i] = from_16(static_cast<const uint16_t *>(segs.param[s])[j], f16 != 0);
    m[i] = 0.0f;
    v[i] = 0.0f;
  }
}

}  // namespace qlora
