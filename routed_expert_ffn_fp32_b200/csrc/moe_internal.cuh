// Internal declarations of the MXFP4 routed-MoE library (sm_100a).
//
// Device helpers shared by the kernels, the workspace layout, and the launch
// functions each kernel file provides to the C-ABI layer (moe_abi.cu).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "moe.h"

namespace moe {

constexpr int kMaxExperts = 1024;
constexpr int kMaxTopK = 16;
constexpr unsigned kFull = 0xffffffffu;
// Row-block mma.sync GEMV: largest batch it takes (larger ones use the K-split
// GEMV), CTAs (one per SM, at most), warps per CTA, tokens per pass.
constexpr int kLaneMaxT = 512;
constexpr int kLaneMaxCtas = 160;
#ifndef MOE_LANE_WARPS
#define MOE_LANE_WARPS 11
#endif
#ifndef MOE_LANE_RMAX
#define MOE_LANE_RMAX 8
#endif
constexpr int kLaneWarps = MOE_LANE_WARPS;
constexpr int kLaneRMax = MOE_LANE_RMAX;
// Per-virtual-expert tables of the row-block GEMV's work split (tokens, passes
// before v, cost units before v, plan, offsets): virtual experts + 1 entries.
constexpr int kLanePfxMax = 258;

// ---------------------------------------------------------------------------
// Workspace layout.  Every region starts on a 256-byte boundary.
// ---------------------------------------------------------------------------
struct WsLayout {
  size_t err;       // int32[16]: [0] status, [1] detail
  size_t counters;  // uint32[16]: arrival counters, zero between calls
  size_t logits;    // f32 [T, E]
  size_t idx;       // i32 [T, k]
  size_t w;         // f32 [T, k]
  size_t counts;    // i32 [E]
  size_t offsets;   // i32 [E + 1]
  size_t entries;   // i32 [T * k]
  size_t plan;      // i32 [E + 2]: [0] active experts, [1..] their ids (ascending)
  size_t xh;        // f16 [T, H]  token rows as f16 (MXFP4-rounded in that mode)
  size_t h;         // [T*k + S*T] rows of 4I bytes: SwiGLU output by pair index (f32, or f16 hi then f16 lo in the row-block GEMV)
  size_t partial;   // f32 [T*k + S*T, H]   expert output rows (by pair index)
  // row-block GEMV (T <= kLaneMaxT)
  size_t lane_part;  // f32 [warps][kLaneRMax][2][32]  split row-block partial sums
  size_t lane_cnt;   // u32 [row blocks]  split row-block atom counts: zero between calls,
                     //     every call leaves them zero
  // tensor-core path only
  size_t xq, xs;    // u8 [rows, H/2], [rows, H/32]  MXFP4 token rows, bucket order
  size_t hq, hs;    // u8 [rows, I/2], [rows, I/32]  MXFP4 SwiGLU rows, bucket order
  size_t item_off;  // i32 [2][E + 2]  work-item prefix sums of the two GEMM phases
  size_t total;
};

inline size_t align256(size_t v) { return (v + 255) & ~size_t(255); }
__host__ __device__ inline size_t align_up16(size_t v) { return (v + 15) & ~size_t(15); }

inline WsLayout ws_layout(const moe_shape_t& s, int has_shared, int gemm) {
  WsLayout L{};
  const size_t T = s.T, H = s.H, I = s.I, E = s.E, k = s.k;
  const size_t rows = T * k + (has_shared ? T : 0);
  size_t o = 0;
  auto take = [&](size_t bytes) { size_t at = o; o = align256(o + bytes); return at; };
  L.err = take(64);
  L.counters = take(64);
  L.logits = take(T * E * 4);
  L.idx = take(T * k * 4);
  L.w = take(T * k * 4);
  L.counts = take(E * 4);
  L.offsets = take((E + 1) * 4);
  L.entries = take(T * k * 4);
  L.plan = take((E + 2) * 4);
  L.xh = take(T * H * 2);
  L.h = take(rows * I * 4);
  L.partial = take(rows * H * 4);
  const bool lane = T <= size_t(kLaneMaxT);
  L.lane_part = take(lane ? size_t(kLaneMaxCtas) * kLaneWarps * kLaneRMax * 2 * 32 * 4 : 0);
  // passes: at most one per virtual expert plus one per kLaneRMax rows
  const size_t passes = E + 1 + (rows + kLaneRMax - 1) / kLaneRMax;
  const size_t rb0 = I / 32, rb1 = H / 32;  // row blocks of the two phases
  L.lane_cnt = take(lane ? passes * (rb0 > rb1 ? rb0 : rb1) * 4 : 0);
  if (gemm) {
    L.xq = take(rows * H / 2);
    L.xs = take(rows * H / 32);
    L.hq = take(rows * I / 2);
    L.hs = take(rows * I / 32);
    L.item_off = take(2 * (E + 2) * 4);
  } else {
    L.xq = L.xs = L.hq = L.hs = L.item_off = o;
  }
  L.total = o;
  return L;
}

// ---------------------------------------------------------------------------
// Device helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ void latch_error(int* err, int code, int detail) {
  if (atomicCAS(err, 0, code) == 0) atomicExch(err + 1, detail);
}

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t b) {
  return __uint_as_float(b << 16);
}

// E8M0 scale byte -> 2^(s-127) as float32.  s = 0 is the subnormal 2^-127,
// s = 255 is NaN (OCP MX v1.0, E8M0).
__device__ __forceinline__ float e8m0_to_f32(uint32_t s) {
  uint32_t bits = s << 23;
  bits = (s == 0u) ? 0x00400000u : bits;
  bits = (s == 255u) ? 0x7fc00000u : bits;
  return __uint_as_float(bits);
}

// Four bytes of E2M1 pairs -> four f16x2 registers (hardware cvt, sm_100a).
// Byte j (bits 8j..8j+7) holds elements 2j (low nibble) and 2j+1 (high
// nibble); out[j] holds them as (low half, high half).
__device__ __forceinline__ void e2m1x8_to_f16x2(uint32_t w, uint32_t (&out)[4]) {
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
      "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
      "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
      : "=r"(out[0]), "=r"(out[1]), "=r"(out[2]), "=r"(out[3])
      : "r"(w));
}

// acc += w.lo * x.lo + w.hi * x.hi with f16 inputs and an f32 accumulator:
// each product is exact and is added to acc with one f32 rounding.
__device__ __forceinline__ float fma2_f16_f32(uint32_t w2, uint32_t x2, float acc) {
  asm("{\n\t.reg .f16 wl, wh, xl, xh;\n\t"
      "mov.b32 {wl, wh}, %1;\n\t"
      "mov.b32 {xl, xh}, %2;\n\t"
      "fma.rn.f32.f16 %0, wl, xl, %0;\n\t"
      "fma.rn.f32.f16 %0, wh, xh, %0;\n\t}"
      : "+f"(acc)
      : "r"(w2), "r"(x2));
  return acc;
}

__device__ __forceinline__ float2 f16x2_to_f32x2(uint32_t v) {
  __half2 h = *reinterpret_cast<__half2*>(&v);
  return __half22float2(h);
}

__device__ __forceinline__ uint32_t f32x2_to_f16x2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Two floats -> one byte of two E2M1 codes (lo -> low nibble), RNE, saturating.
__device__ __forceinline__ uint32_t f32x2_to_e2m1x2(float lo, float hi) {
  uint32_t out;
  asm("{\n\t.reg .b8 r;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 r, %2, %1;\n\t"
      "cvt.u32.u8 %0, r;\n\t}"
      : "=r"(out)
      : "f"(lo), "f"(hi));
  return out;
}

// Streaming 16-byte load that does not allocate in L1 (weights are read once).
__device__ __forceinline__ uint4 ldg_stream(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ uint32_t ldg_u8(const uint8_t* p) {
  return static_cast<uint32_t>(__ldg(p));
}

// Programmatic dependent launch: wait for the preceding kernel's memory, then
// let the next kernel's blocks be scheduled.  Both are no-ops without PDL.
__device__ __forceinline__ void pdl_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" :::);
}

// MXFP4 scale exponent of a block from its largest magnitude (OCP MX v1.0:
// X = floor(log2 amax) - emax(E2M1) with emax = 2, clamped to [-127, 127];
// amax = 0 gives -127).
__device__ __forceinline__ int mx_scale_exponent(float amax) {
  const uint32_t bits = __float_as_uint(amax) & 0x7fffffffu;
  const int ef = int(bits >> 23);  // biased exponent; 0 for zero and subnormals
  const int X = ef - 127 - 2;     // ef = 0: zero or subnormal, below the clamp
  return X < -127 ? -127 : (X > 127 ? 127 : X);
}

// 2^e as a float for e in [-127, 127] (e = -127 is the subnormal 2^-127).
__device__ __forceinline__ float exp2i(int e) {
  return e >= -126 ? __uint_as_float(uint32_t(e + 127) << 23) : __uint_as_float(0x00400000u);
}

// 32 bf16 values -> 32 f16 values (exact for |v| >= 2^-17 and |v| <= 65504);
// with mx the block is first rounded through MXFP4 (OCP scale, RNE, saturate).
__device__ __forceinline__ void bf16_block_to_f16(const uint16_t* src, uint16_t* dst, bool mx) {
  float f[32];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint4 v = *reinterpret_cast<const uint4*>(src + 8 * q);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      f[8 * q + 2 * j] = bf16_bits_to_f32(w[j] & 0xffffu);
      f[8 * q + 2 * j + 1] = bf16_bits_to_f32(w[j] >> 16);
    }
  }
  if (mx) {
    float amax = 0.f;
#pragma unroll
    for (int j = 0; j < 32; ++j) amax = fmaxf(amax, fabsf(f[j]));
    const int X = mx_scale_exponent(amax);
    const float inv = exp2i(-X), sc = exp2i(X);
#pragma unroll
    for (int j = 0; j < 32; j += 8) {
      uint32_t byte4 = 0;
#pragma unroll
      for (int b = 0; b < 4; ++b)
        byte4 |= f32x2_to_e2m1x2(f[j + 2 * b] * inv, f[j + 2 * b + 1] * inv) << (8 * b);
      uint32_t h2[4];
      e2m1x8_to_f16x2(byte4, h2);
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const float2 d = f16x2_to_f32x2(h2[b]);
        f[j + 2 * b] = d.x * sc;
        f[j + 2 * b + 1] = d.y * sc;
      }
    }
  }
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint4 o;
    o.x = f32x2_to_f16x2(f[8 * q + 0], f[8 * q + 1]);
    o.y = f32x2_to_f16x2(f[8 * q + 2], f[8 * q + 3]);
    o.z = f32x2_to_f16x2(f[8 * q + 4], f[8 * q + 5]);
    o.w = f32x2_to_f16x2(f[8 * q + 6], f[8 * q + 7]);
    *reinterpret_cast<uint4*>(dst + 8 * q) = o;
  }
}

// ---------------------------------------------------------------------------
// Kernel argument blocks
// ---------------------------------------------------------------------------
struct ExpertPtrs {
  const uint8_t* gq;
  const uint8_t* gs;
  const uint8_t* uq;
  const uint8_t* us;
  const uint8_t* dq;
  const uint8_t* ds;
};

struct RouteArgs {
  const uint16_t* x;
  uint16_t* xh;       // optional: f16 copy of x written by the router (decode path)
  int act_mxfp4;      // round xh through MXFP4 first
  const float* w_router;
  const float* bias;
  float* logits;
  int32_t* idx;
  float* w;
  int32_t* counts;
  int32_t* offsets;
  int32_t* entries;
  int32_t* plan;
  uint32_t* counter;
  int* err;
  int has_shared;
  int T, H, E, k;
};

struct FfnArgs {
  ExpertPtrs ex;
  ExpertPtrs sh;  // shared expert (n = 1) when has_shared
  const uint16_t* x;
  const uint16_t* xh;   // f16 token rows [T, H] (decode path)
  const int32_t* offsets;
  const int32_t* entries;
  const int32_t* plan;
  const float* topk_w;  // down kernel with combine
  float* h;             // [rows, I]
  float* partial;       // [rows, H]
  uint16_t* y;          // combine output or nullptr
  int* err;
  int T, H, I, E, k;
  int has_shared;
  int act_mxfp4;
};

// ---------------------------------------------------------------------------
// Virtual experts of the FFN kernels: v < plan[0] is the v-th active routed
// expert (its bucket rows), v = plan[0] the shared expert (all T tokens).
// ---------------------------------------------------------------------------
struct VExpert {
  const uint8_t* q[2];
  const uint8_t* s[2];
  const int32_t* rows;  // pair indices of the bucket, or nullptr for the shared expert
  int R;                // tokens
};

__device__ __forceinline__ VExpert vexpert(const FfnArgs& a, int phase, int v, int nA) {
  VExpert ve;
  const int K = phase == 0 ? a.H : a.I;
  const int ROWS = phase == 0 ? a.I : a.H;
  const size_t mat = size_t(ROWS) * (K / 2), smat = size_t(ROWS) * (K / 32);
  if (v < nA) {
    const int e = a.plan[1 + v];
    const int beg = a.offsets[e], end = a.offsets[e + 1];
    ve.rows = a.entries + beg;
    ve.R = end - beg;
    if (phase == 0) {
      ve.q[0] = a.ex.gq + e * mat; ve.s[0] = a.ex.gs + e * smat;
      ve.q[1] = a.ex.uq + e * mat; ve.s[1] = a.ex.us + e * smat;
    } else {
      ve.q[0] = a.ex.dq + e * mat; ve.s[0] = a.ex.ds + e * smat;
      ve.q[1] = nullptr; ve.s[1] = nullptr;
    }
  } else {
    ve.rows = nullptr;
    ve.R = a.T;
    if (phase == 0) {
      ve.q[0] = a.sh.gq; ve.s[0] = a.sh.gs;
      ve.q[1] = a.sh.uq; ve.s[1] = a.sh.us;
    } else {
      ve.q[0] = a.sh.dq; ve.s[0] = a.sh.ds;
      ve.q[1] = nullptr; ve.s[1] = nullptr;
    }
  }
  return ve;
}

// Output row (pair index, or T*k + t for the shared expert) of bucket row r.
__device__ __forceinline__ int out_row(const FfnArgs& a, const VExpert& ve, int r) {
  return ve.rows ? ve.rows[r] : a.T * a.k + r;
}
__device__ __forceinline__ int token_of(const FfnArgs& a, const VExpert& ve, int r) {
  return ve.rows ? ve.rows[r] / a.k : r;
}

// ---------------------------------------------------------------------------
// Launchers (return cudaError_t of the launch)
// ---------------------------------------------------------------------------
struct DeviceInfo {
  int sm_count;
  int max_smem_optin;
};
DeviceInfo device_info();

cudaError_t launch_route_logits(const RouteArgs& a, bool fuse_tail, cudaStream_t st);
size_t route_fused_smem(int T, int H, int E, int k);
cudaError_t launch_topk(const RouteArgs& a, cudaStream_t st);
cudaError_t launch_bucket(const RouteArgs& a, cudaStream_t st);
cudaError_t launch_plan(const RouteArgs& a, cudaStream_t st);

cudaError_t launch_ffn_gemv(const FfnArgs& a, cudaStream_t st);
// Lane-per-row GEMV of both phases; cudaErrorNotSupported when the shape does
// not fit it (the caller then uses launch_ffn_gemv).
cudaError_t launch_ffn_lane(const FfnArgs& a, float* lane_part, uint32_t* lane_cnt,
                            cudaStream_t st);
bool lane_supported(const moe_shape_t& s);
cudaError_t launch_x_f16(const uint16_t* x, int T, int H, int act_mxfp4, uint16_t* xh,
                         cudaStream_t st);

struct GemmBuffers {
  uint8_t* xq;
  uint8_t* xs;
  uint8_t* hq;
  uint8_t* hs;
  int32_t* item_off0;
  int32_t* item_off1;
};
bool gemm_supported(const moe_shape_t& s);
cudaError_t launch_ffn_gemm(const FfnArgs& a, const GemmBuffers& gb, cudaStream_t st);
cudaError_t launch_combine(const float* partial, const float* w, int T, int H, int k,
                           int has_shared, uint16_t* y, cudaStream_t st);
cudaError_t launch_act_quant(const float* in, int rows, int K, uint8_t* q, uint8_t* s,
                             cudaStream_t st);
cudaError_t launch_decode(const uint8_t* q, const uint8_t* s, int rows, int K, float* out,
                          cudaStream_t st);

// Launch helper: every kernel goes out with programmatic stream serialisation
// so its blocks can be scheduled while the previous kernel drains; each
// kernel calls pdl_wait() before its first global memory access.
template <typename Kernel, typename... Args>
cudaError_t launch_pdl(Kernel kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

}  // namespace moe
