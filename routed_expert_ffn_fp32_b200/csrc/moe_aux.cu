// MXFP4 block decode (for tests) and MXFP4 activation quantisation.
//
// Element format: OCP Microscaling v1.0 MXFP4, the format of the routed
// experts in the "ds4-ssd" README ("Run SSD Sidecar Mode").  The activation
// quantiser follows the same specification's scale rule
// (2^(floor(log2 amax) - 2) per 32 values) with round-to-nearest-even onto the
// E2M1 grid and saturation, as used by the MXFP4 activation mode.
#include "moe_internal.cuh"

namespace moe {
namespace {

__global__ void __launch_bounds__(256) k_decode(const uint8_t* q, const uint8_t* s, long long nblk,
                                                float* out) {
  pdl_wait();
  pdl_trigger();
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= nblk) return;
  const uint4 c = *reinterpret_cast<const uint4*>(q + i * 16);
  // the scale through the same hardware ue8m0 conversion the row-block GEMV uses
  const float sc = __uint_as_float(ue8m0x2_to_bf16x2(uint32_t(s[i])) << 16);
  const uint32_t w[4] = {c.x, c.y, c.z, c.w};
  float4* o = reinterpret_cast<float4*>(out + i * 32);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    uint32_t h[4];
    e2m1x8_to_f16x2(w[j], h);
    const float2 a = f16x2_to_f32x2(h[0]), b = f16x2_to_f32x2(h[1]);
    const float2 c2 = f16x2_to_f32x2(h[2]), d = f16x2_to_f32x2(h[3]);
    o[2 * j] = make_float4(a.x * sc, a.y * sc, b.x * sc, b.y * sc);
    o[2 * j + 1] = make_float4(c2.x * sc, c2.y * sc, d.x * sc, d.y * sc);
  }
}

__global__ void __launch_bounds__(256) k_act_quant(const float* in, long long nblk, uint8_t* q,
                                                   uint8_t* s) {
  pdl_wait();
  pdl_trigger();
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= nblk) return;
  const float4* p = reinterpret_cast<const float4*>(in + i * 32);
  float f[32];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const float4 v = __ldg(p + j);
    f[4 * j] = v.x;
    f[4 * j + 1] = v.y;
    f[4 * j + 2] = v.z;
    f[4 * j + 3] = v.w;
  }
  float amax = 0.f;
#pragma unroll
  for (int j = 0; j < 32; ++j) amax = fmaxf(amax, fabsf(f[j]));
  const int X = mx_scale_exponent(amax);
  const float inv = exp2i(-X);
  uint32_t word[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    uint32_t acc = 0;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const int e = 8 * j + 2 * b;
      acc |= f32x2_to_e2m1x2(f[e] * inv, f[e + 1] * inv) << (8 * b);
    }
    word[j] = acc;
  }
  *reinterpret_cast<uint4*>(q + i * 16) = make_uint4(word[0], word[1], word[2], word[3]);
  s[i] = uint8_t(X + 127);
}

__global__ void k_set_words(uint32_t* words, uint32_t w0, uint32_t w1) {
  pdl_wait();
  pdl_trigger();
  words[0] = w0;
  words[1] = w1;
}

}  // namespace

cudaError_t launch_set_words(uint32_t* words, uint32_t w0, uint32_t w1, cudaStream_t st) {
  return launch_pdl(k_set_words, dim3(1), dim3(1), 0, st, words, w0, w1);
}

cudaError_t launch_decode(const uint8_t* q, const uint8_t* s, int rows, int K, float* out,
                          cudaStream_t st) {
  const long long nblk = (long long)rows * (K / 32);
  if (nblk == 0) return cudaSuccess;
  return launch_pdl(k_decode, dim3(unsigned((nblk + 255) / 256)), dim3(256), 0, st, q, s, nblk,
                    out);
}

cudaError_t launch_act_quant(const float* in, int rows, int K, uint8_t* q, uint8_t* s,
                             cudaStream_t st) {
  const long long nblk = (long long)rows * (K / 32);
  if (nblk == 0) return cudaSuccess;
  return launch_pdl(k_act_quant, dim3(unsigned((nblk + 255) / 256)), dim3(256), 0, st, in, nblk,
                    q, s);
}

}  // namespace moe
