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
constexpr int kLaneWarps = 10;
constexpr int kLaneRMax = 8;
// Per-virtual-expert tables of the row-block GEMV's work split (tokens, passes
// before v, cost units before v, plan, offsets): virtual experts + 1 entries.
constexpr int kLanePfxMax = 258;

// ---------------------------------------------------------------------------
// Workspace layout.  Every region starts on a 256-byte boundary.
// ---------------------------------------------------------------------------
// Words of the error region: [0] status, [1] detail, [2] wait limit in
// microseconds (0: kDefaultWaitUs), [3] debug switches (MOE_DEBUG_*).
constexpr unsigned kDefaultWaitUs = 2000000u;

struct WsLayout {
  size_t err;       // int32[16]: status, detail, wait limit, debug switches
  size_t counters;  // uint32[16]: arrival counters, zero between calls
  size_t logits;    // f32 [T, E]
  size_t idx;       // i32 [T, k]
  size_t w;         // f32 [T, k]
  size_t counts;    // i32 [E]
  size_t offsets;   // i32 [E + 1]
  size_t entries;   // i32 [T * k]
  size_t plan;      // i32 [E + 2]: [0] active experts, [1..] their ids (ascending)
  size_t xh;        // f16 [T, H]  token rows as f16, row t scaled by 2^-s_t (MXFP4-rounded first in that mode)
  size_t xexp;      // u8 [T]      s_t + 127
  size_t h;         // [T*k + S*T] rows of h_pitch(I) bytes: SwiGLU output by pair index (f32 [I] on
                    //             the K-split GEMV; f16 hi [I], f16 lo [I], block exponents on the
                    //             row-block GEMV)
  size_t partial;   // f32 [T*k + S*T, H]   expert output rows (by pair index)
  // row-block GEMV (T <= kLaneMaxT)
  size_t lane_part;  // f32 [warps][kLaneRMax][2][32]  split row-block partial sums
  size_t lane_cnt;   // u32 [row blocks]  split row-block atom counts, cleared by the kernel that
                     //     writes the f16 token rows, before every call's GEMV
  // tensor-core path only
  size_t xq, xs;    // u8 [rows, H/2], [rows, H/32]  MXFP4 token rows, bucket order
  size_t hq, hs;    // u8 [rows, I/2], [rows, I/32]  MXFP4 SwiGLU rows, bucket order
  size_t item_off;  // i32 [2][E + 2]  work-item prefix sums of the two GEMM phases
  size_t total;
};

inline size_t align256(size_t v) { return (v + 255) & ~size_t(255); }
__host__ __device__ inline size_t align_up16(size_t v) { return (v + 15) & ~size_t(15); }

// Bytes of one h row: f16 hi [I], f16 lo [I], then one exponent byte per
// 32-value block, padded to 16 bytes (at least the I float32 values of the
// K-split GEMV).
__host__ __device__ inline size_t h_pitch(size_t I) { return 4 * I + align_up16(I / 32); }

// Split-block counters of the row-block GEMV: one per row block of the larger
// phase and per pass (at most one pass per virtual expert plus one per
// kLaneRMax rows).
inline size_t lane_cnt_words(const moe_shape_t& s, int has_shared) {
  const size_t rows = size_t(s.T) * s.k + (has_shared ? s.T : 0);
  const size_t passes = size_t(s.E) + 1 + (rows + kLaneRMax - 1) / kLaneRMax;
  const size_t rb0 = size_t(s.I) / 32, rb1 = size_t(s.H) / 32;
  return passes * (rb0 > rb1 ? rb0 : rb1);
}

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
  L.xexp = take(T);
  L.h = take(rows * h_pitch(I));
  L.partial = take(rows * H * 4);
  const bool lane = T <= size_t(kLaneMaxT);
  L.lane_part = take(lane ? size_t(kLaneMaxCtas) * kLaneWarps * kLaneRMax * 2 * 32 * 4 : 0);
  L.lane_cnt = take(lane ? lane_cnt_words(s, has_shared) * 4 : 0);
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

// Exponent s of the power-of-two scale of a token row's f16 copy, from the
// row's largest bf16 magnitude (bits with the sign cleared): the row is stored
// as x * 2^-s with its largest magnitude in [1, 2).  Every element down to
// 2^-17 of that magnitude keeps its 8 significant bits (f16 subnormals start
// at 2^-24), and no product of a weight with a scaled value exceeds twice the
// weight, so the scaled sums overflow float32 only where sums of the weights'
// magnitudes would.  s lies in [-126, 127]; a row of zeros, or one holding an
// infinity or NaN, gets s = 0.
__device__ __forceinline__ int row_f16_exponent(uint32_t amax_bf16_bits) {
  if (amax_bf16_bits == 0u || amax_bf16_bits >= 0x7f80u) return 0;
  const int field = int(amax_bf16_bits >> 7);  // bf16 exponent field; 0 for subnormals
  return field == 0 ? -126 : field - 127;
}

// Largest magnitude of 8 bf16 values (16 bytes), as bf16 bits with the sign
// cleared, folded into m (per-halfword unsigned max).
__device__ __forceinline__ uint32_t bf16x8_absmax(const uint4& v, uint32_t m) {
  m = __vmaxu2(m, v.x & 0x7fff7fffu);
  m = __vmaxu2(m, v.y & 0x7fff7fffu);
  m = __vmaxu2(m, v.z & 0x7fff7fffu);
  m = __vmaxu2(m, v.w & 0x7fff7fffu);
  return m;
}

// Two E8M0 scale bytes (low 16 bits of w) -> two bf16 powers of two
// 2^(s-127) (low byte -> low half).  The conversion keeps the format's special
// values: byte 0 is the subnormal 2^-127, byte 255 is NaN.
__device__ __forceinline__ uint32_t ue8m0x2_to_bf16x2(uint32_t w) {
  uint32_t r;
  asm("{\n\t.reg .b16 lo;\n\tmov.b32 {lo, _}, %1;\n\tcvt.rn.bf16x2.ue8m0x2 %0, lo;\n\t}"
      : "=r"(r)
      : "r"(w));
  return r;
}

// 32 bf16 values -> 32 f16 values of v * inv, inv = 2^-s from
// row_f16_exponent (exact for every element within 2^-17 of the row's largest
// magnitude); with mx the block is first rounded through MXFP4 (OCP scale,
// RNE, saturate) in float32.
__device__ __forceinline__ void bf16_block_to_f16(const uint16_t* src, uint16_t* dst, bool mx,
                                                  float inv) {
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
    const float qinv = exp2i(-X > 127 ? 127 : -X), sc = exp2i(X);
#pragma unroll
    for (int j = 0; j < 32; j += 8) {
      uint32_t byte4 = 0;
#pragma unroll
      for (int b = 0; b < 4; ++b)
        byte4 |= f32x2_to_e2m1x2(f[j + 2 * b] * qinv, f[j + 2 * b + 1] * qinv) << (8 * b);
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
    o.x = f32x2_to_f16x2(f[8 * q + 0] * inv, f[8 * q + 1] * inv);
    o.y = f32x2_to_f16x2(f[8 * q + 2] * inv, f[8 * q + 3] * inv);
    o.z = f32x2_to_f16x2(f[8 * q + 4] * inv, f[8 * q + 5] * inv);
    o.w = f32x2_to_f16x2(f[8 * q + 6] * inv, f[8 * q + 7] * inv);
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
  uint16_t* xh;       // optional: scaled f16 copy of x written by the router (decode path)
  uint8_t* xexp;      // with xh: per-row scale exponents s_t + 127
  int act_mxfp4;      // round xh through MXFP4 first
  uint32_t* cnt_clear;  // with xh: the row-block GEMV's split-block counters, zeroed here
  int cnt_words;
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
  // optional scratch for the prefill router's K-split partial logits
  // (f32 [splits][T][E]); null: one split, logits written directly
  float* lpart;
  size_t lpart_bytes;
};

struct FfnArgs {
  ExpertPtrs ex;
  ExpertPtrs sh;  // shared expert (n = 1) when has_shared
  const uint16_t* x;
  const uint16_t* xh;   // scaled f16 token rows [T, H] (decode path)
  const uint8_t* xexp;  // their scale exponents s_t + 127 [T]
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
// Scaled f16 token rows and their exponents for the row-block GEMV; also zeroes
// cnt_words split-block counters at cnt_clear (may be 0 / nullptr).
cudaError_t launch_x_f16(const uint16_t* x, int T, int H, int act_mxfp4, uint16_t* xh,
                         uint8_t* xexp, uint32_t* cnt_clear, int cnt_words, cudaStream_t st);

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
cudaError_t launch_combine_range(const float* partial, const float* w, const int32_t* idx,
                                 int e_begin, int e_end, int T, int H, int k, int has_shared,
                                 float* y, cudaStream_t st);
cudaError_t launch_round_bf16(const float* in, long long n, uint16_t* out, cudaStream_t st);
cudaError_t launch_act_quant(const float* in, int rows, int K, uint8_t* q, uint8_t* s,
                             cudaStream_t st);
// words[0] = w0, words[1] = w1 (one thread; ordered on the stream).
cudaError_t launch_set_words(uint32_t* words, uint32_t w0, uint32_t w1, cudaStream_t st);
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
