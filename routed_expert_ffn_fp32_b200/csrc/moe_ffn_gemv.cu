// Grouped GEMV over the activated MXFP4 experts (decode / verify batches).
//
// Only the experts some token chose are read (ainews.cool "antirez ds4
// DeepSeek Metal inference", 技术深度解析: block-sparse matmul that loads only
// activated experts' weights; "ds4-ssd" README, "Run SSD Sidecar Mode":
// MXFP4 routed experts).  Each projection row is dequantised in registers:
// a lane loads one 16-byte chunk = one 32-element MX block (so one E8M0
// scale per lane per row), converts the E2M1 pairs with the sm_100a
// cvt.rn.f16x2.e2m1x2 instruction, multiplies by the token rows held in
// registers and accumulates in float32; the block's power-of-two scale is
// applied once to the block sum.
//
// Work split ("virtual experts"): v < nA is the v-th activated routed expert
// (ascending id, from the bucket's plan); v == nA is the shared expert when
// present.  A projection's rows of all virtual experts form one list of
// nV * ROWS units; every CTA of the persistent grid takes an equal contiguous
// range of it, so HBM traffic is spread evenly over the SMs whatever the
// routing.  Phase 0 (gate/up): ROWS = I, each unit is gate row i and up row i,
// the epilogue writes h = silu(g) * u.  Phase 1 (down): ROWS = H, each unit is
// one output row d, the epilogue writes the expert output into `partial`.
//
// Inside a CTA (4 warps) the K dimension of a row is split over KS warps
// (KS = 1, 2 or 4, 32*KS lanes cover the row's blocks); the 4/KS warp groups
// work on different units.  A warp accumulates UG units x NPROJ projections x
// RC tokens, then one butterfly "transpose" reduction over its 32 lanes
// leaves one finished value per lane (31 shuffles for 32 values instead of
// 5 per value); the KS warps' partial sums are added in shared memory.
#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;

// Arithmetic policies for one 32-element block dot product.
enum Policy : int {
  kMixed = 0,  // x in f16; fma.rn.f32.f16 (exact f16 products, f32 accumulate)
  kF32x2 = 1,  // x in f32; weights widened to f32; packed fma.rn.f32x2
};

template <int POL>
struct XReg;
template <>
struct XReg<kMixed> {
  uint32_t v[16];  // f16x2 pairs (x[2j], x[2j+1])
};
template <>
struct XReg<kF32x2> {
  float2 v[16];
};

__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  unsigned long long ra, rb, rc, rd;
  ra = (static_cast<unsigned long long>(__float_as_uint(a.y)) << 32) | __float_as_uint(a.x);
  rb = (static_cast<unsigned long long>(__float_as_uint(b.y)) << 32) | __float_as_uint(b.x);
  rc = (static_cast<unsigned long long>(__float_as_uint(c.y)) << 32) | __float_as_uint(c.x);
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(rd) : "l"(ra), "l"(rb), "l"(rc));
  return make_float2(__uint_as_float(uint32_t(rd)), __uint_as_float(uint32_t(rd >> 32)));
}

// 32 float values of a block -> the policy's register form.  With act_mxfp4
// the block is first quantised to MXFP4 and dequantised (OCP MX v1.0 scale
// 2^(floor(log2 amax) - 2), RNE onto E2M1, saturating), which is exactly the
// value an MXFP4 activation operand carries.
template <int POL>
__device__ __forceinline__ void pack_block(float (&f)[32], bool act_mxfp4, XReg<POL>& out) {
  if (act_mxfp4) {
    float amax = 0.f;
#pragma unroll
    for (int j = 0; j < 32; ++j) amax = fmaxf(amax, fabsf(f[j]));
    const int X = mx_scale_exponent(amax);
    const float inv = exp2i(-X > 127 ? 127 : -X);
    const float sc = exp2i(X);
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
  for (int j = 0; j < 16; ++j) {
    if constexpr (POL == kMixed) out.v[j] = f32x2_to_f16x2(f[2 * j], f[2 * j + 1]);
    else out.v[j] = make_float2(f[2 * j], f[2 * j + 1]);
  }
}

__device__ __forceinline__ void load_block_bf16(const uint16_t* row, int b, float (&f)[32]) {
  const uint4* p = reinterpret_cast<const uint4*>(row + size_t(b) * 32);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint4 v = __ldg(p + q);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      f[8 * q + 2 * j] = bf16_bits_to_f32(w[j] & 0xffffu);
      f[8 * q + 2 * j + 1] = bf16_bits_to_f32(w[j] >> 16);
    }
  }
}

__device__ __forceinline__ void load_block_f32(const float* row, int b, float (&f)[32]) {
  const float4* p = reinterpret_cast<const float4*>(row + size_t(b) * 32);
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const float4 v = __ldcg(p + q);  // written by the previous kernel: bypass L1
    f[4 * q] = v.x;
    f[4 * q + 1] = v.y;
    f[4 * q + 2] = v.z;
    f[4 * q + 3] = v.w;
  }
}

__device__ __forceinline__ void decode_codes(const uint4& c, uint32_t (&h)[16]) {
  uint32_t t[4];
  e2m1x8_to_f16x2(c.x, t);
  h[0] = t[0]; h[1] = t[1]; h[2] = t[2]; h[3] = t[3];
  e2m1x8_to_f16x2(c.y, t);
  h[4] = t[0]; h[5] = t[1]; h[6] = t[2]; h[7] = t[3];
  e2m1x8_to_f16x2(c.z, t);
  h[8] = t[0]; h[9] = t[1]; h[10] = t[2]; h[11] = t[3];
  e2m1x8_to_f16x2(c.w, t);
  h[12] = t[0]; h[13] = t[1]; h[14] = t[2]; h[15] = t[3];
}

template <int POL>
__device__ __forceinline__ float block_dot(const uint32_t (&w)[16], const XReg<POL>& x) {
  if constexpr (POL == kMixed) {
    float a0 = 0.f, a1 = 0.f;  // two chains for latency
#pragma unroll
    for (int j = 0; j < 16; j += 2) {
      a0 = fma2_f16_f32(w[j], x.v[j], a0);
      a1 = fma2_f16_f32(w[j + 1], x.v[j + 1], a1);
    }
    return a0 + a1;
  } else {
    float2 a = make_float2(0.f, 0.f);
#pragma unroll
    for (int j = 0; j < 16; ++j) a = ffma2(f16x2_to_f32x2(w[j]), x.v[j], a);
    return a.x + a.y;
  }
}

// Butterfly reduce-scatter of NVAL per-lane values over the warp: afterwards
// every lane holds the warp total of value index (lane & (NVAL - 1)).
template <int NVAL>
__device__ __forceinline__ float transpose_reduce(float (&v)[NVAL], int lane) {
#pragma unroll
  for (int m = NVAL / 2; m >= 1; m >>= 1) {
    const bool upper = (lane & m) != 0;
#pragma unroll
    for (int i = 0; i < m; ++i) {
      const float keep = upper ? v[i + m] : v[i];
      const float send = upper ? v[i] : v[i + m];
      v[i] = keep + __shfl_xor_sync(kFull, send, m);
    }
  }
#pragma unroll
  for (int m = NVAL; m < 32; m <<= 1) v[0] += __shfl_xor_sync(kFull, v[0], m);
  return v[0];
}

// ---------------------------------------------------------------------------
// Asynchronous global -> shared copies (cp.async): each lane streams its own
// 16-byte code chunks into a per-warp ring of stages, so several stages of
// weights are in flight while the warp computes on an earlier one.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async8(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(smem_u32(dst)), "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async4(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)), "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void group_barrier(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

constexpr int kStages = 3;        // ring depth per warp
constexpr int kSlots = 8;         // 512-byte code chunks per stage per warp
constexpr int kChunk = 512;       // one warp-wide 16-byte-per-lane row slice
constexpr int kStageBytes = kSlots * (kChunk + 32);
constexpr int kRingBytes = kStages * kStageBytes;
constexpr int kPartBytes = 2 * kWarps * 32 * 4;
constexpr int kGemvSmem = kWarps * kRingBytes + kPartBytes;

template <int PHASE>
struct PhaseCfg {
  static constexpr int NPROJ = PHASE == 0 ? 2 : 1;
  // Both projections take their inputs as float32 (bf16 token rows and the
  // float32 SwiGLU output are exact there, over the whole bf16 range), with
  // the weights widened to float32 and packed float32 FMAs.
  static constexpr int POL = kF32x2;
};

struct Worker {
  int KS, NG, grp, gl, lstride, nb, bar_id, bar_n;
  int warp, lane;
  unsigned char* ring;  // this warp's stages
  float* part;          // [2][kWarps][32]
  int fast_scales;      // scale rows 4-byte aligned: stage them with cp.async
  unsigned parity;      // stage counter (selects the part buffer)
};

// One virtual expert, units [r0, r1), tokens [t0, t0 + nt) of its bucket.
template <int PHASE, int BPL, int RC>
__device__ void run_segment(const FfnArgs& a, const VExpert& ve, int r0, int r1, int t0, int nt,
                            Worker& wk) {
  using C = PhaseCfg<PHASE>;
  constexpr int NPROJ = C::NPROJ;
  constexpr int POL = C::POL;
  constexpr int UG_SM = kSlots / (NPROJ * BPL) > 0 ? kSlots / (NPROJ * BPL) : 1;
  constexpr int UG_ACC = 32 / (NPROJ * RC) > 0 ? 32 / (NPROJ * RC) : 1;
  constexpr int UG = UG_SM < UG_ACC ? UG_SM : UG_ACC;
  constexpr int NVAL = UG * NPROJ * RC;
  static_assert((NVAL & (NVAL - 1)) == 0 && NVAL <= 32, "NVAL must be a power of two <= 32");
  const int K = PHASE == 0 ? a.H : a.I;
  const size_t rowq = size_t(K) / 2;
  const int nb = wk.nb, lane = wk.lane;
  const int nunits = r1 - r0;
  const int nst = (nunits + UG - 1) / UG;
  const int span0 = (wk.warp % wk.KS) * 32;  // first block of this warp's K slice

  auto issue = [&](int st) {
    if (st < nst) {
      unsigned char* stage = wk.ring + (st % kStages) * kStageBytes;
#pragma unroll
      for (int u = 0; u < UG; ++u) {
        const int row = r0 + st * UG + u;
        if (row < r1) {
#pragma unroll
          for (int pj = 0; pj < NPROJ; ++pj) {
#pragma unroll
            for (int m = 0; m < BPL; ++m) {
              const int slot = (u * NPROJ + pj) * BPL + m;
              const int b = wk.gl + m * wk.lstride;
              if (b < nb)
                cp_async16(stage + slot * kChunk + lane * 16,
                           ve.q[pj] + size_t(row) * rowq + size_t(b) * 16);
              if (wk.fast_scales) {
                const int sb = span0 + m * wk.lstride;  // first block of the 32-byte span
                if (lane < 8 && sb + 4 * lane + 4 <= nb)
                  cp_async4(stage + kSlots * kChunk + slot * 32 + lane * 4,
                            ve.s[pj] + size_t(row) * nb + sb + 4 * lane);
              }
            }
          }
        }
      }
    }
    cp_async_commit();
  };

#pragma unroll
  for (int s = 0; s < kStages - 1; ++s) issue(s);

  // token rows -> registers (overlaps the first stages in flight)
  XReg<POL> xr[BPL][RC];
#pragma unroll
  for (int m = 0; m < BPL; ++m) {
    const int b = wk.gl + m * wk.lstride;
#pragma unroll
    for (int t = 0; t < RC; ++t) {
      float f[32];
      if (t < nt && b < nb) {
        const int r = t0 + t;
        if constexpr (PHASE == 0) {
          load_block_bf16(a.x + size_t(token_of(a, ve, r)) * a.H, b, f);
        } else {
          load_block_f32(a.h + size_t(out_row(a, ve, r)) * a.I, b, f);
        }
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) f[j] = 0.f;
      }
      pack_block<POL>(f, a.act_mxfp4 != 0, xr[m][t]);
    }
  }

  for (int st = 0; st < nst; ++st) {
    issue(st + kStages - 1);
    cp_async_wait<kStages - 1>();
    __syncwarp();
    const unsigned char* stage = wk.ring + (st % kStages) * kStageBytes;
    float acc[NVAL];
#pragma unroll
    for (int i = 0; i < NVAL; ++i) acc[i] = 0.f;
#pragma unroll
    for (int u = 0; u < UG; ++u) {
      if (r0 + st * UG + u < r1) {
#pragma unroll
        for (int pj = 0; pj < NPROJ; ++pj) {
#pragma unroll
          for (int m = 0; m < BPL; ++m) {
            const int slot = (u * NPROJ + pj) * BPL + m;
            const int b = wk.gl + m * wk.lstride;
            if (b < nb) {
              const uint4 c = *reinterpret_cast<const uint4*>(stage + slot * kChunk + lane * 16);
              const int row = r0 + st * UG + u;
              const uint32_t sbyte =
                  wk.fast_scales ? uint32_t(stage[kSlots * kChunk + slot * 32 + lane])
                                 : ldg_u8(ve.s[pj] + size_t(row) * nb + b);
              uint32_t w[16];
              decode_codes(c, w);
              const float sc = e8m0_to_f32(sbyte);
#pragma unroll
              for (int t = 0; t < RC; ++t) {
                const float bs = block_dot<POL>(w, xr[m][t]);
                float& dst = acc[(u * NPROJ + pj) * RC + t];
                dst = fmaf(sc, bs, dst);
              }
            }
          }
        }
      }
    }
    const float tot = transpose_reduce<NVAL>(acc, lane);
    float* part = wk.part + (wk.parity & 1u) * (kWarps * 32);
    if (lane < NVAL) part[wk.warp * 32 + lane] = tot;
    group_barrier(wk.bar_id, wk.bar_n);
    // finalize: the KS warps of the group add their K-slice sums
    const int q = (wk.warp % wk.KS) * 32 + lane;
    if (q < UG * RC) {
      const int u = q / RC, t = q % RC;
      const int row = r0 + st * UG + u;
      if (row < r1 && t < nt) {
        float s0 = 0.f, s1 = 0.f;
        for (int w = 0; w < wk.KS; ++w) {
          const float* pw = part + (wk.grp * wk.KS + w) * 32;
          s0 += pw[(u * NPROJ + 0) * RC + t];
          if constexpr (NPROJ == 2) s1 += pw[(u * NPROJ + 1) * RC + t];
        }
        const int orow = out_row(a, ve, t0 + t);
        if constexpr (PHASE == 0) {
          a.h[size_t(orow) * a.I + row] = s0 / (1.f + expf(-s0)) * s1;  // silu(g) * u
        } else {
          a.partial[size_t(orow) * a.H + row] = s0;
        }
      }
    }
    ++wk.parity;
  }
  cp_async_wait<0>();
  __syncwarp();
}

// Four CTAs per SM, or two where the float32 operand registers of BPL * RCMAX
// blocks per lane would not fit the register budget of four.
template <int PHASE, int BPL, int RCMAX>
__global__ void __launch_bounds__(kThreads, BPL * RCMAX >= 4 ? 2 : 4)
    k_ffn_gemv(FfnArgs a, int KS, int fast_scales) {
  extern __shared__ __align__(128) unsigned char smem[];
  pdl_wait();
  pdl_trigger();
  Worker wk;
  wk.lane = threadIdx.x & 31;
  wk.warp = threadIdx.x >> 5;
  wk.KS = KS;
  wk.NG = kWarps / KS;
  wk.grp = wk.warp / KS;
  wk.gl = (wk.warp % KS) * 32 + wk.lane;
  wk.lstride = 32 * KS;
  wk.nb = (PHASE == 0 ? a.H : a.I) / 32;
  wk.bar_id = 1 + wk.grp;
  wk.bar_n = 32 * KS;
  wk.ring = smem + wk.warp * kRingBytes;
  wk.part = reinterpret_cast<float*>(smem + kWarps * kRingBytes);
  wk.fast_scales = fast_scales;
  wk.parity = 0;

  const int nA = a.plan[0];
  const int nV = nA + (a.has_shared ? 1 : 0);
  const int ROWS = PHASE == 0 ? a.I : a.H;
  const long long U = (long long)nV * ROWS;
  const long long nW = (long long)gridDim.x * wk.NG;
  const long long worker = (long long)blockIdx.x * wk.NG + wk.grp;
  const long long ub = U * worker / nW;
  const long long ue = U * (worker + 1) / nW;
  long long u = ub;
  while (u < ue) {
    const int v = int(u / ROWS);
    const int r0 = int(u % ROWS);
    const int r1 = int(min((long long)ROWS, r0 + (ue - u)));
    const VExpert ve = vexpert(a, PHASE, v, nA);
    for (int t0 = 0; t0 < ve.R; t0 += RCMAX) {
      const int nt = min(RCMAX, ve.R - t0);
      if (RCMAX >= 2 && nt == 2) {
        run_segment<PHASE, BPL, (RCMAX >= 2 ? 2 : 1)>(a, ve, r0, r1, t0, nt, wk);
      } else {
        run_segment<PHASE, BPL, 1>(a, ve, r0, r1, t0, nt, wk);
      }
    }
    u += r1 - r0;
  }
}

// K split and blocks per lane for a projection of K columns.
inline void split_of(int K, int& KS, int& BPL) {
  const int nb = K / 32;
  if (nb <= 32) { KS = 1; BPL = 1; }
  else if (nb <= 64) { KS = 2; BPL = 1; }
  else if (nb <= 128) { KS = 4; BPL = 1; }
  else if (nb <= 256) { KS = 4; BPL = 2; }
  else { KS = 4; BPL = 4; }
}

// Largest token tile per pass: x registers hold BPL * RC blocks per lane.
// Token rows per pass: two at most (their registers stay small enough for
// four CTAs per SM); a bucket of more tokens takes several passes over the
// same weights, the later ones served from L2.
inline int rcmax_of(int PHASE, int T, int BPL) {
  (void)PHASE;
  return (T >= 2 && BPL <= 2) ? 2 : 1;
}

template <int PHASE, int BPL, int RCMAX>
cudaError_t launch_one(const FfnArgs& a, int grid, int KS, int fast, cudaStream_t st) {
  auto kern = k_ffn_gemv<PHASE, BPL, RCMAX>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kGemvSmem);
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, dim3(grid), dim3(kThreads), size_t(kGemvSmem), st, a, KS, fast);
}

template <int PHASE>
cudaError_t launch_phase(const FfnArgs& a, int grid, cudaStream_t st) {
  const int K = PHASE == 0 ? a.H : a.I;
  int KS, BPL;
  split_of(K, KS, BPL);
  const int RCMAX = rcmax_of(PHASE, a.T, BPL);
  const int fast = (K / 32) % 4 == 0;
#define MOE_GEMV_CASE(B, R) \
  if (BPL == B && RCMAX == R) return launch_one<PHASE, B, R>(a, grid, KS, fast, st);
  MOE_GEMV_CASE(1, 1)
  MOE_GEMV_CASE(1, 2)
  MOE_GEMV_CASE(2, 1)
  MOE_GEMV_CASE(2, 2)
  MOE_GEMV_CASE(4, 1)
#undef MOE_GEMV_CASE
  return cudaErrorInvalidValue;
}

__global__ void __launch_bounds__(256) k_combine(const float* partial, const float* w, int T,
                                                 int H, int k, int has_shared, uint16_t* y) {
  pdl_wait();
  pdl_trigger();
  const int per_row = H / 4;
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (long long)T * per_row) return;
  const int t = int(i / per_row), c = int(i % per_row) * 4;
  float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int j = 0; j < k; ++j) {
    const float wj = __ldcg(w + size_t(t) * k + j);
    const float4 p = __ldcg(reinterpret_cast<const float4*>(partial + (size_t(t) * k + j) * H + c));
    s.x = fmaf(wj, p.x, s.x);
    s.y = fmaf(wj, p.y, s.y);
    s.z = fmaf(wj, p.z, s.z);
    s.w = fmaf(wj, p.w, s.w);
  }
  if (has_shared) {
    const float4 p =
        __ldcg(reinterpret_cast<const float4*>(partial + (size_t(T) * k + t) * H + c));
    s.x += p.x;
    s.y += p.y;
    s.z += p.z;
    s.w += p.w;
  }
  __nv_bfloat162 lo = __floats2bfloat162_rn(s.x, s.y), hi = __floats2bfloat162_rn(s.z, s.w);
  uint2 out;
  out.x = *reinterpret_cast<uint32_t*>(&lo);
  out.y = *reinterpret_cast<uint32_t*>(&hi);
  *reinterpret_cast<uint2*>(y + size_t(t) * H + c) = out;
}

// Float32 combine of the pairs whose expert lies in [e_begin, e_end) (the
// experts one rank of an expert-parallel group holds): the same slot-order
// sums as k_combine, left in float32 for a sum over ranks.
__global__ void __launch_bounds__(256) k_combine_range(const float* partial, const float* w,
                                                       const int32_t* idx, int e_begin, int e_end,
                                                       int T, int H, int k, int has_shared,
                                                       float* y) {
  pdl_wait();
  pdl_trigger();
  const int per_row = H / 4;
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (long long)T * per_row) return;
  const int t = int(i / per_row), c = int(i % per_row) * 4;
  float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int j = 0; j < k; ++j) {
    const int e = __ldg(idx + size_t(t) * k + j);
    if (e < e_begin || e >= e_end) continue;
    const float wj = __ldg(w + size_t(t) * k + j);
    const float4 p = __ldcg(reinterpret_cast<const float4*>(partial + (size_t(t) * k + j) * H + c));
    s.x = fmaf(wj, p.x, s.x);
    s.y = fmaf(wj, p.y, s.y);
    s.z = fmaf(wj, p.z, s.z);
    s.w = fmaf(wj, p.w, s.w);
  }
  if (has_shared) {
    const float4 p =
        __ldcg(reinterpret_cast<const float4*>(partial + (size_t(T) * k + t) * H + c));
    s.x += p.x;
    s.y += p.y;
    s.z += p.z;
    s.w += p.w;
  }
  *reinterpret_cast<float4*>(y + size_t(t) * H + c) = s;
}

// float32 -> bf16 (round to nearest even), four values per thread.
__global__ void __launch_bounds__(256) k_round_bf16(const float* in, long long n4, uint16_t* out) {
  pdl_wait();
  pdl_trigger();
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n4) return;
  const float4 v = __ldcg(reinterpret_cast<const float4*>(in) + i);
  __nv_bfloat162 lo = __floats2bfloat162_rn(v.x, v.y), hi = __floats2bfloat162_rn(v.z, v.w);
  uint2 o;
  o.x = *reinterpret_cast<uint32_t*>(&lo);
  o.y = *reinterpret_cast<uint32_t*>(&hi);
  reinterpret_cast<uint2*>(out)[i] = o;
}

// bf16 token rows -> scaled f16 rows and their exponents (for calls that do
// not route through the fused router): one warp per token row finds the
// row's largest magnitude, then converts its 32-value blocks.  The grid also
// zeroes the row-block GEMV's split-block counters.
__global__ void __launch_bounds__(256) k_x_f16(const uint16_t* x, int T, int H, int act_mxfp4,
                                               uint16_t* xh, uint8_t* xexp, uint32_t* cnt,
                                               int cnt_words) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int nthr = gridDim.x * blockDim.x;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < cnt_words; i += nthr) cnt[i] = 0u;
  const int nwarps = nthr / 32;
  for (int t = (blockIdx.x * blockDim.x + threadIdx.x) / 32; t < T; t += nwarps) {
    const uint16_t* row = x + size_t(t) * H;
    uint32_t m = 0;
    for (int i = lane; i < H / 8; i += 32) m = bf16x8_absmax(__ldg(reinterpret_cast<const uint4*>(row) + i), m);
    m = max(m & 0xffffu, m >> 16);
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) m = max(m, __shfl_xor_sync(kFull, m, off));
    const int sx = row_f16_exponent(m);
    if (lane == 0) xexp[t] = uint8_t(sx + 127);
    const float inv = exp2i(-sx);
    for (int b = lane; b < H / 32; b += 32)
      bf16_block_to_f16(row + size_t(b) * 32, xh + size_t(t) * H + size_t(b) * 32, act_mxfp4 != 0,
                        inv);
  }
}

}  // namespace

cudaError_t launch_x_f16(const uint16_t* x, int T, int H, int act_mxfp4, uint16_t* xh,
                         uint8_t* xexp, uint32_t* cnt_clear, int cnt_words, cudaStream_t st) {
  const int by_rows = (T + 7) / 8;
  const int by_cnt = (cnt_words + 255) / 256;
  const int grid = max(1, min(1024, max(by_rows, by_cnt)));
  return launch_pdl(k_x_f16, dim3(grid), dim3(256), 0, st, x, T, H, act_mxfp4, xh, xexp,
                    cnt_clear, cnt_clear ? cnt_words : 0);
}

int gemv_grid() {
  static int occ = 0;
  if (occ == 0) {
    int o = 0;
    cudaFuncSetAttribute(k_ffn_gemv<0, 1, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         kGemvSmem);
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&o, k_ffn_gemv<0, 1, 2>, kThreads, kGemvSmem);
    occ = o > 0 ? o : 1;
  }
  return device_info().sm_count * occ;
}

cudaError_t launch_ffn_gemv(const FfnArgs& a, cudaStream_t st) {
  const cudaError_t e = launch_phase<0>(a, gemv_grid(), st);
  if (e != cudaSuccess) return e;
  return launch_phase<1>(a, gemv_grid(), st);
}

cudaError_t launch_combine(const float* partial, const float* w, int T, int H, int k,
                           int has_shared, uint16_t* y, cudaStream_t st) {
  const long long n = (long long)T * (H / 4);
  const int blocks = int((n + 255) / 256);
  return launch_pdl(k_combine, dim3(blocks), dim3(256), 0, st, partial, w, T, H, k, has_shared,
                    y);
}

cudaError_t launch_combine_range(const float* partial, const float* w, const int32_t* idx,
                                 int e_begin, int e_end, int T, int H, int k, int has_shared,
                                 float* y, cudaStream_t st) {
  const long long n = (long long)T * (H / 4);
  const int blocks = int((n + 255) / 256);
  return launch_pdl(k_combine_range, dim3(blocks), dim3(256), 0, st, partial, w, idx, e_begin, e_end,
                    T, H, k, has_shared, y);
}

cudaError_t launch_round_bf16(const float* in, long long n, uint16_t* out, cudaStream_t st) {
  const long long n4 = n / 4;
  if (n4 == 0) return cudaSuccess;
  return launch_pdl(k_round_bf16, dim3(unsigned((n4 + 255) / 256)), dim3(256), 0, st, in, n4, out);
}

}  // namespace moe
