// AdamW step for the LoRA adapters, for states paged out to host memory.
//
// «QLoRA는 어떻게 65B 모델을 GPU 한 장에 올렸나», § "메모리 회계: 세 겹의 최적화"
// (Paged Optimizer): only A and B are trained; Adam's m and v may overflow to
// CPU pinned memory, and running the update beside the backward on another
// CUDA stream hides most of the transfer. Here the update itself runs on the
// GPU: m and v (and, if the caller wants, the fp32 master copy) may be device
// memory or pinned host memory that the GPU reaches directly over the
// interconnect, so a paged state costs one read and one write of 8 bytes per
// parameter across the link and nothing else. The step is a pure stream
// (about 22 bytes per parameter in total), vectorised 4 wide.
//
// Update (AdamW, decoupled weight decay, bias-corrected, t 1-based):
//   m <- b1 m + (1 - b1) g;  v <- b2 v + (1 - b2) g^2
//   p <- p (1 - lr wd);      p <- p - (lr / (1 - b1^t)) m / (sqrt(v) / sqrt(1 - b2^t) + eps)
// and the bf16 copy the GEMMs read, if given, becomes bf16(p).
#include "kernels.h"
#include "ptx.cuh"

namespace qlora {

namespace {

__device__ __forceinline__ float adamw_one(float p, float g, float& m, float& v, const AdamwParams& a) {
  m = fmaf(a.beta1, m, (1.0f - a.beta1) * g);
  v = fmaf(a.beta2, v, (1.0f - a.beta2) * g * g);
  p = p * a.decay;
  const float denom = sqrtf(v) * a.inv_sqrt_bc2 + a.eps;
  return p - a.step_size * (m / denom);
}

}  // namespace

__global__ void __launch_bounds__(256) k_adamw(AdamwParams a) {
  const int64_t n4 = a.n >> 2;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (a.vec4) {
    for (int64_t i = t0; i < n4; i += stride) {
      float4 p = reinterpret_cast<const float4*>(a.master)[i];
      const float4 g = __ldcs(reinterpret_cast<const float4*>(a.grad) + i);
      float4 m = reinterpret_cast<const float4*>(a.m)[i];
      float4 v = reinterpret_cast<const float4*>(a.v)[i];
      p.x = adamw_one(p.x, g.x, m.x, v.x, a);
      p.y = adamw_one(p.y, g.y, m.y, v.y, a);
      p.z = adamw_one(p.z, g.z, m.z, v.z, a);
      p.w = adamw_one(p.w, g.w, m.w, v.w, a);
      reinterpret_cast<float4*>(a.master)[i] = p;
      reinterpret_cast<float4*>(a.m)[i] = m;
      reinterpret_cast<float4*>(a.v)[i] = v;
      if (a.param != nullptr) {
        uint2 o;
        o.x = pack_bf16x2(p.x, p.y);
        o.y = pack_bf16x2(p.z, p.w);
        reinterpret_cast<uint2*>(a.param)[i] = o;
      }
    }
  }
  // elements not covered by the 4-wide loop (all of them when unaligned)
  for (int64_t i = (a.vec4 ? n4 * 4 : 0) + t0; i < a.n; i += stride) {
    float m = a.m[i], v = a.v[i];
    const float p = adamw_one(a.master[i], a.grad[i], m, v, a);
    a.master[i] = p;
    a.m[i] = m;
    a.v[i] = v;
    if (a.param != nullptr) a.param[i] = __float2bfloat16_rn(p);
  }
}

}  // namespace qlora
