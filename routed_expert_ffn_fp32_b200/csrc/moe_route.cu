// Router logits, softmax / top-k / renormalise, and the stable bucket of
// (token, slot) pairs by expert.
//
// The pages only say that a token activates a few experts (ainews.cool
// "antirez ds4 DeepSeek Metal inference", 技术深度解析: top-k routing over
// fine-grained experts) and that k is a run-time knob ("ds4-ssd" README,
// "Experimental Pro Support": --moe-expert-topk).  Formulas used here:
//   logits[t,e] = sum_h x[t,h] W_r[e,h] + b[e]           (float32)
//   idx[t,:]    = the k largest logits, descending, ties to the lower index
//   w[t,j]      = exp(l_j - l_0) / sum_{j'<k} exp(l_j' - l_0)
// which equals softmax over all E followed by renormalisation over the k.
//
// Kernels
//   k_route_logits<TT>: one CTA per (2 experts, 1 token) or per (1 expert,
//     TT > 1 tokens).  Eight warps: with two experts warp w takes expert w / 4
//     and the w % 4 quarter of H, with one expert the w-th eighth of H; each
//     lane streams float4 router rows and keeps TT float32 partial sums.  The
//     bf16 token rows sit in shared memory; the f16 copy of the token rows
//     for the row-block GEMV is written from there by all CTAs of a token tile,
//     32 values per thread.  Every product meets at most H/128 + 9 roundings
//     (lane chain, 5 shuffle levels, 3 sums of the warps' parts -- a chain of
//     quarters or a tree of eighths -- and the bias), the bound the parity
//     tests use for near-ties.
//     With fuse_tail the CTA that finishes last (arrival counter in the
//     workspace, reset to zero by that CTA) runs top-k (a warp per token) and
//     a one-warp bucket for the whole batch, so a decode step routes in one
//     launch.
//   k_route_logits_tiled: batches of more than 32 tokens (see the kernel).
//   k_topk: one warp per token.
//   k_bucket: one CTA; counts by shared-memory atomics, exclusive scan, then a
//     stable placement of each 1024-pair chunk: ranks among equal experts come
//     from __match_any_sync inside a warp plus per-warp counts of earlier warps.
//     Batches of more than 2048 pairs take k_bucket_count + k_bucket_place,
//     one CTA per 2048 pairs, with the same result.
#include <float.h>

#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int kRouteThreads = 256;
constexpr int kBucketThreads = 1024;

// ----------------------------------------------------------------- top-k ---
template <int NV>
__device__ void topk_warp(const float* row, int E, int k, int32_t* idx_out, float* w_out,
                          int32_t* idx_smem) {
  const int lane = threadIdx.x & 31;
  float v[NV];
  uint32_t removed = 0;
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const int e = lane + 32 * i;
    float val = -FLT_MAX;
    if (e < E) {
      val = __ldcg(row + e);
      if (val != val) val = -INFINITY;  // NaN ranks lowest
    } else {
      removed |= 1u << i;
    }
    v[i] = val;
  }
  float my_v = -INFINITY;
  int my_i = 0;
  for (int j = 0; j < k; ++j) {
    float bv = -INFINITY;
    int bi = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const int e = lane + 32 * i;
      const bool live = !((removed >> i) & 1u);
      if (live && (v[i] > bv || (v[i] == bv && e < bi))) {
        bv = v[i];
        bi = e;
      }
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) {
      const float ov = __shfl_xor_sync(kFull, bv, off);
      const int oi = __shfl_xor_sync(kFull, bi, off);
      if (ov > bv || (ov == bv && oi < bi)) {
        bv = ov;
        bi = oi;
      }
    }
    if ((bi & 31) == lane) removed |= 1u << (bi >> 5);
    if (lane == j) {
      my_v = bv;
      my_i = bi;
    }
  }
  const float vmax = __shfl_sync(kFull, my_v, 0);
  float p = (lane < k) ? expf(my_v - vmax) : 0.f;
  float sum = p;
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) sum += __shfl_xor_sync(kFull, sum, off);
  if (lane < k) {
    idx_out[lane] = my_i;
    w_out[lane] = p / sum;
    if (idx_smem) idx_smem[lane] = my_i;
  }
}

template <typename F>
__device__ void dispatch_nv(int E, F&& f) {
  if (E <= 32) f.template operator()<1>();
  else if (E <= 64) f.template operator()<2>();
  else if (E <= 128) f.template operator()<4>();
  else if (E <= 256) f.template operator()<8>();
  else if (E <= 512) f.template operator()<16>();
  else f.template operator()<32>();
}

__device__ void topk_block(const RouteArgs& a, int32_t* idx_smem) {
  const int warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  for (int t = warp; t < a.T; t += nwarps) {
    const float* row = a.logits + size_t(t) * a.E;
    int32_t* is = idx_smem ? idx_smem + t * a.k : nullptr;
    dispatch_nv(a.E, [&]<int NV>() {
      topk_warp<NV>(row, a.E, a.k, a.idx + size_t(t) * a.k, a.w + size_t(t) * a.k, is);
    });
  }
}

// ---------------------------------------------------------------- bucket ---
struct BucketSmem {
  int* cnt;       // [E]
  int* cur;       // [E]
  int* wsum;      // [2 * 33]
  uint8_t* hist;  // [nwarps * E]
};

__device__ __forceinline__ BucketSmem bucket_smem(void* base, int E, int nwarps) {
  BucketSmem s;
  s.cnt = reinterpret_cast<int*>(base);
  s.cur = s.cnt + E;
  s.wsum = s.cur + E;
  s.hist = reinterpret_cast<uint8_t*>(s.wsum + 2 * 33);
  (void)nwarps;
  return s;
}

inline size_t bucket_smem_bytes(int E, int nthreads) {
  return size_t(E) * 8 + 2 * 33 * 4 + size_t(nthreads / 32) * E;
}

// Block-wide exclusive scan of per-thread (a, b) pairs; returns the exclusive
// prefix of each and writes the totals.
__device__ __forceinline__ void block_scan2(int a, int b, int& ea, int& eb, int& ta, int& tb,
                                            int* wsum) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  int ia = a, ib = b;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int ua = __shfl_up_sync(kFull, ia, off), ub = __shfl_up_sync(kFull, ib, off);
    if (lane >= off) {
      ia += ua;
      ib += ub;
    }
  }
  if (lane == 31) {
    wsum[warp] = ia;
    wsum[33 + warp] = ib;
  }
  __syncthreads();
  if (warp == 0) {
    int va = lane < nwarps ? wsum[lane] : 0, vb = lane < nwarps ? wsum[33 + lane] : 0;
    int sa = va, sb = vb;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int ua = __shfl_up_sync(kFull, sa, off), ub = __shfl_up_sync(kFull, sb, off);
      if (lane >= off) {
        sa += ua;
        sb += ub;
      }
    }
    if (lane < nwarps) {
      wsum[lane] = sa - va;  // exclusive warp prefix
      wsum[33 + lane] = sb - vb;
    }
    if (lane == 31) {
      wsum[32] = sa;
      wsum[65] = sb;
    }
  }
  __syncthreads();
  ea = wsum[warp] + ia - a;
  eb = wsum[33 + warp] + ib - b;
  ta = wsum[32];
  tb = wsum[65];
  __syncthreads();
}

// counts[] -> offsets[] / plan[] (active experts ascending); also primes cur[].
// Null outputs are skipped.
__device__ void offsets_and_plan(const int* cnt, int E, int32_t* counts, int32_t* offsets,
                                 int32_t* plan, int* cur, int* wsum) {
  const int nthreads = blockDim.x, tid = threadIdx.x;
  const int per = (E + nthreads - 1) / nthreads;
  const int beg = min(E, tid * per), end = min(E, beg + per);
  int local = 0, lact = 0;
  for (int e = beg; e < end; ++e) {
    local += cnt[e];
    lact += cnt[e] > 0;
  }
  int ex, eact, total, tact;
  block_scan2(local, lact, ex, eact, total, tact, wsum);
  for (int e = beg; e < end; ++e) {
    const int c = cnt[e];
    if (counts) counts[e] = c;
    if (offsets) offsets[e] = ex;
    if (cur) cur[e] = ex;
    if (c > 0 && plan) plan[1 + eact++] = e;
    ex += c;
  }
  if (tid == 0) {
    if (offsets) offsets[E] = total;
    if (plan) plan[0] = tact;
  }
}

// Stable placement of pairs [p0, p1) in chunks of the block's size: the next
// free entry of expert e is s.cur[e] (advanced here); ranks among equal
// experts come from __match_any_sync inside a warp plus per-warp counts of
// earlier warps (s.hist, zero on entry and on exit).
__device__ void place_pairs(const int32_t* idx, int p0, int p1, int E, int32_t* entries,
                            BucketSmem s) {
  const int tid = threadIdx.x, nthreads = blockDim.x;
  const int lane = tid & 31, warp = tid >> 5;
  const unsigned lt_mask = (1u << lane) - 1u;
  for (int base = p0; base < p1; base += nthreads) {
    const int p = base + tid;
    int e = p < p1 ? idx[p] : -1;
    const bool valid = e >= 0 && e < E;
    const unsigned grp = __match_any_sync(kFull, valid ? e : (E + lane));
    const int rank = __popc(grp & lt_mask);
    const int gcnt = __popc(grp);
    if (valid && rank == 0) s.hist[warp * E + e] = uint8_t(gcnt);
    __syncthreads();
    if (valid) {
      int prefix = 0;
      for (int w = 0; w < warp; ++w) prefix += s.hist[w * E + e];
      entries[s.cur[e] + prefix + rank] = p;
    }
    __syncthreads();
    if (valid && rank == 0) {
      atomicAdd(&s.cur[e], gcnt);
      s.hist[warp * E + e] = 0;
    }
    __syncthreads();
  }
}

// Stable counting sort of the npairs pairs by expert; block of any size.
__device__ void bucket_block(const int32_t* idx, int npairs, int E, int32_t* counts,
                             int32_t* offsets, int32_t* entries, int32_t* plan, int* err,
                             BucketSmem s) {
  const int tid = threadIdx.x, nthreads = blockDim.x;
  const int nwarps = nthreads >> 5;
  for (int e = tid; e < E; e += nthreads) s.cnt[e] = 0;
  for (int i = tid; i < nwarps * E; i += nthreads) s.hist[i] = 0;
  __syncthreads();
  for (int p = tid; p < npairs; p += nthreads) {
    const int e = idx[p];
    if (e >= 0 && e < E) atomicAdd(&s.cnt[e], 1);
    else latch_error(err, MOE_ERR_DEVICE_DATA, p);
  }
  __syncthreads();
  offsets_and_plan(s.cnt, E, counts, offsets, plan, s.cur, s.wsum);
  __syncthreads();
  place_pairs(idx, 0, npairs, E, entries, s);
}

// One-warp stable bucket for small batches (the decode tail): counts by
// shared-memory atomics, warp scans over the experts, then pairs placed in
// order, ranks among equal experts from __match_any_sync.  No block barrier.
__device__ int bucket_warp(const int32_t* idx, int npairs, int E, int32_t* counts,
                           int32_t* offsets, int32_t* entries, int32_t* plan, int* err, int* cnt,
                           int* cur) {
  const int lane = threadIdx.x & 31;
  const unsigned lt_mask = (1u << lane) - 1u;
  for (int e = lane; e < E; e += 32) cnt[e] = 0;
  __syncwarp();
  for (int p = lane; p < npairs; p += 32) {
    const int e = idx[p];
    if (e >= 0 && e < E) atomicAdd(&cnt[e], 1);
    else latch_error(err, MOE_ERR_DEVICE_DATA, p);
  }
  __syncwarp();
  int run = 0, run_act = 0;
  for (int base = 0; base < E; base += 32) {
    const int e = base + lane;
    const int c = e < E ? cnt[e] : 0;
    const int act = c > 0;
    int incl = c, incl_act = act;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(kFull, incl, off), ya = __shfl_up_sync(kFull, incl_act, off);
      if (lane >= off) {
        incl += y;
        incl_act += ya;
      }
    }
    if (e < E) {
      const int ex = run + incl - c;
      counts[e] = c;
      offsets[e] = ex;
      cur[e] = ex;
      if (act) plan[1 + run_act + incl_act - 1] = e;
    }
    run += __shfl_sync(kFull, incl, 31);
    run_act += __shfl_sync(kFull, incl_act, 31);
  }
  if (lane == 0) {
    offsets[E] = run;
    plan[0] = run_act;
  }
  __syncwarp();
  for (int base = 0; base < npairs; base += 32) {
    const int p = base + lane;
    const int e = p < npairs ? idx[p] : -1;
    const bool valid = e >= 0 && e < E;
    const unsigned grp = __match_any_sync(kFull, valid ? e : (E + lane));
    const int rank = __popc(grp & lt_mask);
    if (valid) entries[cur[e] + rank] = p;
    __syncwarp();
    if (valid && rank == 0) cur[e] += __popc(grp);
    __syncwarp();
  }
  return run_act;
}

// ---------------------------------------------------------------- kernels ---
template <int TT>
__global__ void __launch_bounds__(kRouteThreads) k_route_logits(RouteArgs a, int fuse_tail) {
  extern __shared__ __align__(16) unsigned char smem[];
  __shared__ int s_exp[TT];
  pdl_wait();
  pdl_trigger();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int H = a.H;
  const int t0 = blockIdx.y * TT;
  const int nt = min(TT, a.T - t0);
  uint16_t* xs = reinterpret_cast<uint16_t*>(smem);                  // [TT][H] bf16
  float* red = reinterpret_cast<float*>(smem + size_t(TT) * H * 2);  // [8][TT]
  // experts per CTA: two for single-token tiles (eight warps split each row
  // in quarters), else one (eighths)
  constexpr int EPC = TT == 1 ? 2 : 1;
  constexpr int PARTS = 8 / EPC;
  const int e = blockIdx.x * EPC + warp / PARTS;
  const int quarter = warp % PARTS;  // this warp's part of the row
  const int qlen = H / PARTS;        // multiple of 4
  const float* wrow = a.w_router + size_t(e < a.E ? e : 0) * H + quarter * qlen;
  // the first eight float4 of this lane's router row go out before the token
  // rows are staged, so the two loads overlap
  float4 wv[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int c = lane * 4 + 128 * j;
    wv[j] = (e < a.E && c < qlen) ? __ldg(reinterpret_cast<const float4*>(wrow + c))
                                  : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  // stage the token rows (16-byte vectors; H % 32 == 0)
  {
    const int vec_per_row = H / 8;
    const uint4* src = reinterpret_cast<const uint4*>(a.x + size_t(t0) * H);
    uint4* dst = reinterpret_cast<uint4*>(xs);
    for (int i = tid; i < nt * vec_per_row; i += kRouteThreads) dst[i] = __ldg(src + i);
  }
  if (a.cnt_clear != nullptr) {
    const int nthr = gridDim.x * gridDim.y * kRouteThreads;
    for (int i = (blockIdx.y * gridDim.x + blockIdx.x) * kRouteThreads + tid; i < a.cnt_words;
         i += nthr)
      a.cnt_clear[i] = 0u;
  }
  __syncthreads();
  if (a.xh != nullptr) {
    // scale exponent of each token row of the tile (one warp per token)
    if (warp < nt) {
      uint32_t m = 0;
      const uint4* row = reinterpret_cast<const uint4*>(xs + size_t(warp) * H);
      for (int i = lane; i < H / 8; i += 32) m = bf16x8_absmax(row[i], m);
      m = max(m & 0xffffu, m >> 16);
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) m = max(m, __shfl_xor_sync(kFull, m, off));
      if (lane == 0) {
        const int sx = row_f16_exponent(m);
        s_exp[warp] = sx;
        if (blockIdx.x == 0) a.xexp[t0 + warp] = uint8_t(sx + 127);
      }
    }
    __syncthreads();
    // scaled f16 copy of the token rows for the expert GEMV: this token
    // tile's 32-value blocks spread over the CTAs of the tile row, one per
    // thread
    const int nblk = nt * (H / 32);
    for (int i = blockIdx.x * kRouteThreads + tid; i < nblk; i += gridDim.x * kRouteThreads) {
      const int t = i / (H / 32), b = i % (H / 32);
      bf16_block_to_f16(xs + size_t(t) * H + 32 * b, a.xh + size_t(t0 + t) * H + 32 * b,
                        a.act_mxfp4 != 0, exp2i(-s_exp[t]));
    }
  }
  float acc[TT];
#pragma unroll
  for (int t = 0; t < TT; ++t) acc[t] = 0.f;
  if (e < a.E) {
    const uint16_t* xq = xs + quarter * qlen;
    // eight float4 loads in flight per lane before the arithmetic on them
    for (int base = lane * 4; base < qlen; base += 128 * 8) {
      if (base != lane * 4) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int c = base + 128 * j;
          wv[j] = c < qlen ? __ldg(reinterpret_cast<const float4*>(wrow + c))
                           : make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int c = base + 128 * j;
        if (c < qlen) {
#pragma unroll
          for (int t = 0; t < TT; ++t) {
            if (t < nt) {
              const uint2 xv = *reinterpret_cast<const uint2*>(xq + size_t(t) * H + c);
              acc[t] = fmaf(bf16_bits_to_f32(xv.x & 0xffffu), wv[j].x, acc[t]);
              acc[t] = fmaf(bf16_bits_to_f32(xv.x >> 16), wv[j].y, acc[t]);
              acc[t] = fmaf(bf16_bits_to_f32(xv.y & 0xffffu), wv[j].z, acc[t]);
              acc[t] = fmaf(bf16_bits_to_f32(xv.y >> 16), wv[j].w, acc[t]);
            }
          }
        }
      }
    }
  }
#pragma unroll
  for (int t = 0; t < TT; ++t) {
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) acc[t] += __shfl_xor_sync(kFull, acc[t], off);
  }
  if (lane == 0) {
#pragma unroll
    for (int t = 0; t < TT; ++t) red[warp * TT + t] = acc[t];
  }
  __syncthreads();
  if (tid < EPC * TT) {
    const int pe = tid / TT, t = tid % TT;
    const int ee = blockIdx.x * EPC + pe;
    if (ee < a.E && t < nt) {
      const float* r = red + (pe * PARTS) * TT + t;
      float s;
      if constexpr (PARTS == 4) {
        s = ((r[0] + r[TT]) + r[2 * TT]) + r[3 * TT];
      } else {
        s = ((r[0] + r[TT]) + (r[2 * TT] + r[3 * TT])) +
            ((r[4 * TT] + r[5 * TT]) + (r[6 * TT] + r[7 * TT]));
      }
      if (a.bias) s += __ldg(a.bias + ee);
      a.logits[size_t(t0 + t) * a.E + ee] = s;
    }
  }
  if (!fuse_tail) return;
  // ---- the last CTA to arrive routes the whole batch ----
  __shared__ int s_last;
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const unsigned total = gridDim.x * gridDim.y;
    s_last = atomicAdd(a.counter, 1u) == total - 1u;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  int32_t* idx_s = reinterpret_cast<int32_t*>(smem);  // reuse: [T*k]
  topk_block(a, idx_s);
  __syncthreads();
  if (warp == 0) {
    int* cnt = reinterpret_cast<int*>(smem + align_up16(size_t(a.T) * a.k * 4));
    bucket_warp(idx_s, a.T * a.k, a.E, a.counts, a.offsets, a.entries, a.plan, a.err, cnt,
                cnt + a.E);
    if (lane == 0) *a.counter = 0u;
  }
}

// Router logits for prefill-sized batches: a 128-token x 64-expert tile per
// CTA over one of S contiguous K ranges (blockIdx.z), K in chunks of 32
// staged in shared memory (double buffered, dynamic), each thread an
// 8-token x 4-expert register tile, two CTAs per SM.  Products of a chunk are
// summed into a fresh register and chunk sums are added to the running total;
// with S > 1 the range sums go to lpart[s] and k_topk adds them in order
// s = 0.., so every product meets at most 32 + H/32 + 1 roundings (the bound
// the parity tests use).
constexpr int kTileT = 128, kTileE = 64, kTileK = 32;
constexpr int kXPitch = kTileT + 4, kWPitch = kTileE + 4;  // floats per k row
constexpr size_t kTiledSmem = size_t(2) * kTileK * (kXPitch + kWPitch) * 4;

__global__ void __launch_bounds__(256, 2) k_route_logits_tiled(RouteArgs a, int S) {
  extern __shared__ __align__(16) float tsm[];
  float* xs = tsm;                              // [2][kTileK][kXPitch]  [k][token]
  float* wsm = tsm + 2 * kTileK * kXPitch;      // [2][kTileK][kWPitch]  [k][expert]
  pdl_wait();
  pdl_trigger();
  const int tid = threadIdx.x;
  const int t0 = blockIdx.y * kTileT, e0 = blockIdx.x * kTileE;
  const int ty = tid / 16, tx = tid % 16;  // tokens ty*8.., experts tx*4..
  const int H = a.H;
  const int nchunks = H / kTileK / S;
  const int kbase = blockIdx.z * nchunks * kTileK;
  // global -> register staging of a chunk: 16 bf16 of one token row and 8
  // floats of one expert row per thread
  const int xr = tid / 2, xc = (tid % 2) * 16;  // token, first k
  const int wr = tid / 4, wc = (tid % 4) * 8;   // expert, first k
  uint4 xreg0, xreg1;
  float4 wreg0, wreg1;
  auto gload = [&](int ck) {
    const int k0 = kbase + ck * kTileK;
    const int t = t0 + xr, e = e0 + wr;
    if (t < a.T) {
      const uint4* px = reinterpret_cast<const uint4*>(a.x + size_t(t) * H + k0 + xc);
      xreg0 = __ldg(px);
      xreg1 = __ldg(px + 1);
    } else {
      xreg0 = xreg1 = make_uint4(0, 0, 0, 0);
    }
    if (e < a.E) {
      const float4* pw = reinterpret_cast<const float4*>(a.w_router + size_t(e) * H + k0 + wc);
      wreg0 = __ldg(pw);
      wreg1 = __ldg(pw + 1);
    } else {
      wreg0 = wreg1 = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  };
  auto sstore = [&](int buf) {
    float* xb = xs + buf * kTileK * kXPitch;
    float* wb = wsm + buf * kTileK * kWPitch;
    const uint32_t xw[8] = {xreg0.x, xreg0.y, xreg0.z, xreg0.w, xreg1.x, xreg1.y, xreg1.z, xreg1.w};
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      xb[(xc + 2 * j) * kXPitch + xr] = bf16_bits_to_f32(xw[j] & 0xffffu);
      xb[(xc + 2 * j + 1) * kXPitch + xr] = bf16_bits_to_f32(xw[j] >> 16);
    }
    const float wv[8] = {wreg0.x, wreg0.y, wreg0.z, wreg0.w, wreg1.x, wreg1.y, wreg1.z, wreg1.w};
#pragma unroll
    for (int j = 0; j < 8; ++j) wb[(wc + j) * kWPitch + wr] = wv[j];
  };
  float acc[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
  gload(0);
  sstore(0);
  __syncthreads();
  for (int ck = 0; ck < nchunks; ++ck) {
    const int buf = ck & 1;
    if (ck + 1 < nchunks) gload(ck + 1);
    const float* xb = xs + buf * kTileK * kXPitch + ty * 8;
    const float* wb = wsm + buf * kTileK * kWPitch + tx * 4;
    float part[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) part[i][j] = 0.f;
#pragma unroll 4
    for (int k = 0; k < kTileK; ++k) {
      const float4 xa = *reinterpret_cast<const float4*>(xb + k * kXPitch);
      const float4 xb4 = *reinterpret_cast<const float4*>(xb + k * kXPitch + 4);
      const float4 wv = *reinterpret_cast<const float4*>(wb + k * kWPitch);
      const float xv[8] = {xa.x, xa.y, xa.z, xa.w, xb4.x, xb4.y, xb4.z, xb4.w};
      const float ww[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) part[i][j] = fmaf(xv[i], ww[j], part[i][j]);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] += part[i][j];
    if (ck + 1 < nchunks) sstore(buf ^ 1);
    __syncthreads();
  }
  float* out = S > 1 ? a.lpart + size_t(blockIdx.z) * a.T * a.E : a.logits;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int t = t0 + ty * 8 + i;
    if (t >= a.T) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int e = e0 + tx * 4 + j;
      if (e < a.E) {
        float v = acc[i][j];
        if (S == 1 && a.bias) v += __ldg(a.bias + e);
        out[size_t(t) * a.E + e] = v;
      }
    }
  }
}

// K splits of the prefill router: the fewest (1, 2, 4, 8, 16) that give every SM
// about six CTAs, within the scratch and with whole 32-value chunks per split
int route_splits(const RouteArgs& a) {
  const long tiles = long((a.E + kTileE - 1) / kTileE) * ((a.T + kTileT - 1) / kTileT);
  const size_t per = size_t(a.T) * a.E * 4;
  int S = 1;
  while (S < 16 && tiles * S < 6L * device_info().sm_count && (a.H / kTileK) % (2 * S) == 0 &&
         a.lpart != nullptr && size_t(2 * S) * per <= a.lpart_bytes)
    S *= 2;
  return S;
}

// The logits row of token t from the router's S K-range sums: all S loads of
// a logit first, then the sums added in range order, then the bias (one warp).
template <int S>
__device__ __forceinline__ void sum_splits(const RouteArgs& a, int t) {
  float* row = a.logits + size_t(t) * a.E;
  const size_t stride = size_t(a.T) * a.E;
#pragma unroll 2
  for (int e = threadIdx.x & 31; e < a.E; e += 32) {
    const float* p = a.lpart + size_t(t) * a.E + e;
    float v[S];
#pragma unroll
    for (int s = 0; s < S; ++s) v[s] = p[s * stride];
    float acc = v[0];
#pragma unroll
    for (int s = 1; s < S; ++s) acc += v[s];
    if (a.bias) acc += __ldg(a.bias + e);
    row[e] = acc;
  }
}

__global__ void __launch_bounds__(kRouteThreads) k_topk(RouteArgs a, int S) {
  pdl_wait();
  pdl_trigger();
  const int warp = threadIdx.x >> 5;
  const int t = blockIdx.x * (kRouteThreads / 32) + warp;
  if (t >= a.T) return;
  if (S > 1) {
    switch (S) {
      case 2: sum_splits<2>(a, t); break;
      case 4: sum_splits<4>(a, t); break;
      case 8: sum_splits<8>(a, t); break;
      default: sum_splits<16>(a, t); break;
    }
    __syncwarp();
  }
  dispatch_nv(a.E, [&]<int NV>() {
    topk_warp<NV>(a.logits + size_t(t) * a.E, a.E, a.k, a.idx + size_t(t) * a.k,
                  a.w + size_t(t) * a.k, nullptr);
  });
}

__global__ void __launch_bounds__(kBucketThreads) k_bucket(RouteArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  pdl_wait();
  pdl_trigger();
  BucketSmem bs = bucket_smem(smem, a.E, kBucketThreads / 32);
  bucket_block(a.idx, a.T * a.k, a.E, a.counts, a.offsets, a.entries, a.plan, a.err, bs);
}

// Multi-CTA stable bucket for large batches (two launches).  CTA c owns the
// pairs [c*kBucketChunk, (c+1)*kBucketChunk).  k_bucket_count: per-CTA counts
// per expert into gcnt[c][E] (shared-memory atomics).  k_bucket_place: every
// CTA adds the counts up in CTA order -- totals and the counts of the CTAs
// before it -- scans the totals into offsets (CTA 0 writes counts, offsets
// and the plan), and places its pairs stably from offset + earlier CTAs'
// counts.  The result equals the one-CTA sort's.
constexpr int kBucketChunk = 2048;

__global__ void __launch_bounds__(kBucketThreads) k_bucket_count(RouteArgs a, int* gcnt) {
  extern __shared__ __align__(16) unsigned char smem[];
  pdl_wait();
  pdl_trigger();
  int* cnt = reinterpret_cast<int*>(smem);
  const int npairs = a.T * a.k;
  const int p0 = blockIdx.x * kBucketChunk, p1 = min(npairs, p0 + kBucketChunk);
  for (int e = threadIdx.x; e < a.E; e += blockDim.x) cnt[e] = 0;
  __syncthreads();
  for (int p = p0 + threadIdx.x; p < p1; p += blockDim.x) {
    const int e = a.idx[p];
    if (e >= 0 && e < a.E) atomicAdd(&cnt[e], 1);
    else latch_error(a.err, MOE_ERR_DEVICE_DATA, p);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < a.E; e += blockDim.x) gcnt[size_t(blockIdx.x) * a.E + e] = cnt[e];
}

__global__ void __launch_bounds__(kBucketThreads) k_bucket_place(RouteArgs a, const int* gcnt) {
  extern __shared__ __align__(16) unsigned char smem[];
  pdl_wait();
  pdl_trigger();
  BucketSmem bs = bucket_smem(smem, a.E, kBucketThreads / 32);
  const int npairs = a.T * a.k;
  const int c = blockIdx.x, nc = gridDim.x;
  // totals (bs.cnt) and the counts of the CTAs before this one (bs.hist is
  // still free: it holds the earlier CTAs' sums until the scan)
  int* before = reinterpret_cast<int*>(bs.hist);
  for (int e = threadIdx.x; e < a.E; e += blockDim.x) {
    int tot = 0, pre = 0;
    for (int j = 0; j < nc; ++j) {
      const int v = gcnt[size_t(j) * a.E + e];
      if (j < c) pre += v;
      tot += v;
    }
    bs.cnt[e] = tot;
    before[e] = pre;
  }
  __syncthreads();
  // every CTA scans the totals into its cursors; CTA 0 also writes the
  // outputs
  if (c == 0) offsets_and_plan(bs.cnt, a.E, a.counts, a.offsets, a.plan, bs.cur, bs.wsum);
  else offsets_and_plan(bs.cnt, a.E, nullptr, nullptr, nullptr, bs.cur, bs.wsum);
  __syncthreads();
  for (int e = threadIdx.x; e < a.E; e += blockDim.x) bs.cur[e] += before[e];
  __syncthreads();
  for (int i = threadIdx.x; i < (kBucketThreads / 32) * a.E; i += blockDim.x) bs.hist[i] = 0;
  __syncthreads();
  const int p0 = c * kBucketChunk, p1 = min(npairs, p0 + kBucketChunk);
  place_pairs(a.idx, p0, p1, a.E, a.entries, bs);
}

// plan[] from caller-provided offsets (component API path).
__global__ void __launch_bounds__(kBucketThreads) k_plan(RouteArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  pdl_wait();
  pdl_trigger();
  int* cnt = reinterpret_cast<int*>(smem);
  int* wsum = cnt + a.E;
  for (int e = threadIdx.x; e < a.E; e += blockDim.x) {
    const int c = __ldg(a.offsets + e + 1) - __ldg(a.offsets + e);
    if (c < 0) latch_error(a.err, MOE_ERR_DEVICE_DATA, e);
    cnt[e] = c < 0 ? 0 : c;
  }
  __syncthreads();
  offsets_and_plan(cnt, a.E, nullptr, nullptr, a.plan, nullptr, wsum);
}

}  // namespace

// ------------------------------------------------------------- launchers ---
static size_t route_smem(int TT, int H) { return size_t(TT) * H * 2 + 8 * TT * 4; }

cudaError_t launch_route_logits(const RouteArgs& a, bool fuse_tail, cudaStream_t st) {
  if (!fuse_tail && a.T > 32) {
    const int S = route_splits(a);
    dim3 grid((a.E + kTileE - 1) / kTileE, (a.T + kTileT - 1) / kTileT, S);
    cudaError_t err = cudaFuncSetAttribute(k_route_logits_tiled,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           int(kTiledSmem));
    if (err != cudaSuccess) return err;
    return launch_pdl(k_route_logits_tiled, grid, dim3(256), kTiledSmem, st, a, S);
  }
  const int TT = a.T <= 1 ? 1 : (a.T <= 2 ? 2 : (a.T <= 4 ? 4 : 8));
  size_t smem = route_smem(TT, a.H);
  if (fuse_tail) {
    const size_t tail = align_up16(size_t(a.T) * a.k * 4) + size_t(a.E) * 8;
    smem = smem > tail ? smem : tail;
  }
  dim3 grid(TT == 1 ? (a.E + 1) / 2 : a.E, (a.T + TT - 1) / TT);
  cudaError_t err = cudaSuccess;
  auto go = [&](auto kern) {
    err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (err == cudaSuccess)
      err = launch_pdl(kern, grid, dim3(kRouteThreads), smem, st, a, int(fuse_tail));
  };
  switch (TT) {
    case 1: go(k_route_logits<1>); break;
    case 2: go(k_route_logits<2>); break;
    case 4: go(k_route_logits<4>); break;
    default: go(k_route_logits<8>); break;
  }
  return err;
}

size_t route_fused_smem(int T, int H, int E, int k) {
  const int TT = T <= 1 ? 1 : (T <= 2 ? 2 : (T <= 4 ? 4 : 8));
  const size_t a = route_smem(TT, H);
  const size_t b = align_up16(size_t(T) * k * 4) + size_t(E) * 8;
  return a > b ? a : b;
}

cudaError_t launch_topk(const RouteArgs& a, cudaStream_t st) {
  const int wpb = kRouteThreads / 32;
  // the split count the tiled router used (one split below its batch sizes)
  const int S = a.T > 32 ? route_splits(a) : 1;
  return launch_pdl(k_topk, dim3((a.T + wpb - 1) / wpb), dim3(kRouteThreads), 0, st, a, S);
}

cudaError_t launch_bucket(const RouteArgs& a, cudaStream_t st) {
  const size_t smem = bucket_smem_bytes(a.E, kBucketThreads);
  const int npairs = a.T * a.k;
  const int nc = (npairs + kBucketChunk - 1) / kBucketChunk;
  const size_t gbytes = size_t(nc) * a.E * 4;
  cudaError_t err;
  if (nc > 1 && a.lpart != nullptr && gbytes <= a.lpart_bytes) {
    // several chunks and scratch for their counts: the two-launch bucket
    int* gcnt = reinterpret_cast<int*>(a.lpart);
    err = launch_pdl(k_bucket_count, dim3(nc), dim3(kBucketThreads), size_t(a.E) * 4, st, a, gcnt);
    if (err != cudaSuccess) return err;
    err = cudaFuncSetAttribute(k_bucket_place, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (err != cudaSuccess) return err;
    return launch_pdl(k_bucket_place, dim3(nc), dim3(kBucketThreads), smem, st, a,
                      static_cast<const int*>(gcnt));
  }
  err = cudaFuncSetAttribute(k_bucket, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (err != cudaSuccess) return err;
  return launch_pdl(k_bucket, dim3(1), dim3(kBucketThreads), smem, st, a);
}

cudaError_t launch_plan(const RouteArgs& a, cudaStream_t st) {
  const size_t smem = size_t(a.E) * 4 + 2 * 33 * 4;
  return launch_pdl(k_plan, dim3(1), dim3(kBucketThreads), smem, st, a);
}

}  // namespace moe
