// dequant.cu -- FP8 block-scaled weights to bf16.
//
// The FP8 form of a weight matrix [rows][cols] is e4m3 bytes q with one fp32 scale s per 128 x 128
// tile (tile [r / 128][c / 128], row-major over ceil(cols / 128) tiles); the weight is q * s.  The
// GEMMs of this library multiply bf16 operands on the tensor cores, so a layer's FP8 matrices are
// expanded to bf16(q * s) (one round-to-nearest-even of the exact product's fp32 rounding) into a
// scratch region of the workspace just before the layer runs.  One launch covers up to five
// matrices; every thread converts groups of 16 consecutive bytes (16 | cols, so a group never
// crosses a tile boundary), reading 16 B and writing 32 B with vector accesses.
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "dg_device.cuh"
#include "dg_kernels.h"

namespace dg {

__device__ __forceinline__ uint32_t fp8x2_to_bf16x2(uint32_t two, float s) {
  const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(two & 0xFFFFu), __NV_E4M3);
  const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h));
  return pack_bf16x2(f.x * s, f.y * s);
}

__device__ __forceinline__ uint4 fp8x8_to_bf16x8(uint2 w, float s) {
  return make_uint4(fp8x2_to_bf16x2(w.x, s), fp8x2_to_bf16x2(w.x >> 16, s), fp8x2_to_bf16x2(w.y, s),
                    fp8x2_to_bf16x2(w.y >> 16, s));
}

__global__ void __launch_bounds__(256) dequant_fp8_kernel(DequantArgs a) {
  pdl_trigger();
  pdl_wait();   // the previous layer's GEMMs may still read the scratch this launch overwrites
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  for (int m = 0; m < a.n; ++m) {
    const DequantMat& t = a.mat[m];
    const uint32_t gpr = (uint32_t)t.cols / 16;           // groups per row
    const size_t n_groups = (size_t)t.rows * gpr;
    const int tc = (t.cols + 127) / 128;
    for (size_t g = (size_t)blockIdx.x * blockDim.x + threadIdx.x; g < n_groups; g += stride) {
      const size_t r = g / gpr;
      const uint32_t c = (uint32_t)(g - r * gpr) * 16u;
      const float s = __ldg(t.s + (r / 128) * tc + c / 128);
      const uint4 q = __ldcs(reinterpret_cast<const uint4*>(t.q + r * t.cols + c));
      uint4* o = reinterpret_cast<uint4*>(t.out + r * t.cols + c);
      o[0] = fp8x8_to_bf16x8(make_uint2(q.x, q.y), s);
      o[1] = fp8x8_to_bf16x8(make_uint2(q.z, q.w), s);
    }
  }
}

cudaError_t dequant_fp8(const DequantArgs& a, int n_sms, cudaStream_t st) {
  if (a.n <= 0) return cudaSuccess;
  return launch_k(dequant_fp8_kernel, dim3(n_sms * 8), dim3(256), 0, st, 1, a);
}

}  // namespace dg
