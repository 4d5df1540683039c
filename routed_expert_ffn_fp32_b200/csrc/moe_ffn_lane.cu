// Lane-per-row GEMV of the expert FFN for small batches (sm_100a).
//
// Computes the same two phases as the other FFN paths (the routed-expert FFN
// of the MoE layer: per routed pair, SwiGLU of the gate/up projections of the
// token, then the down projection), for batches of at most kLaneMaxT tokens
// where every expert sees only a few rows of activations and the work is a
// stream of MXFP4 weights past a handful of token vectors.
//
// Work decomposition.  A projection's weight matrix [ROWS, K] is cut into
// row blocks of 32 rows and, along K, into atoms of 128 values (64 code
// bytes per row).  The atoms of all (virtual expert, pass, row block) triples
// form one flat index space, atom fastest; every warp of the grid takes a
// contiguous range of it of equal cost, an atom of a pass with R tokens
// costing 1 + R (moving and decoding the codes, then R dot products).  One lane owns one row of the block: its dot
// products need no cross-lane reduction, and the token values it multiplies
// with are the same for all 32 lanes (one broadcast load serves the warp).
//
// Data movement.  Each warp keeps D slots of shared memory.  A slot holds the
// 32 x 64-byte code box of an atom per projection, loaded by a TMA tile copy
// (64-byte swizzle, so the 16-byte reads of any 8 consecutive rows fall in
// distinct banks), and the atom's 128 values of each of the pass's tokens,
// loaded by 1-D bulk copies, and each row's 4 scale bytes per projection,
// loaded by the row's lane with cp.async; all complete on the slot's
// mbarrier.  The copy for stage j + D is issued as soon as stage j has been
// consumed.
//
// Tokens.  A pass handles up to kRMax tokens of an expert; an expert with
// more tokens has one row block per pass in the flat index space (its weights
// are streamed once per pass).
//
// Results.  A warp whose range covers a whole row block writes the block's
// outputs directly (phase 0: SwiGLU into h; phase 1: the expert output row).
// A row block split between warps is finished deterministically: each
// contributor stores its partial sums in its own slot (a warp has two, for
// the first and the last block of its range), enters the slot in the block's
// table at the position of its first atom, and adds its atom count to the
// block's counter; the contributor that completes the count adds the slots
// in table order, applies the epilogue and clears the table entries and the
// counter.
//
// Every wait is bounded (globaltimer); on expiry the kernel latches
// MOE_ERR_TIMEOUT, lets its in-flight copies land and returns.
#include <cuda.h>

#include <type_traits>

#include "moe_internal.cuh"

namespace moe {

bool make_tma_map_u8_box(CUtensorMap* m, const void* base, uint64_t row_bytes, uint64_t rows,
                         uint32_t box_bytes, uint32_t box_rows);

namespace {

constexpr int kLW = kLaneWarps;          // warps per CTA, one CTA per SM
constexpr int kLThreads = 32 * kLW;
constexpr int kRMax = kLaneRMax;         // tokens per pass
#ifndef MOE_LANE_ATOM
#define MOE_LANE_ATOM 128
#endif
#ifndef MOE_LANE_SLOTS
#define MOE_LANE_SLOTS 3
#endif
constexpr int kAtomVals = MOE_LANE_ATOM;  // weights of a row per atom (128 or 256)
constexpr int kAtomCode = kAtomVals / 2;  // code bytes of a row per atom (64 or 128)
constexpr int kBlk = kAtomVals / 32;      // scale blocks per atom
constexpr int kBox = 32 * kAtomCode;      // one projection's 32-row box
static_assert(kAtomVals == 128 || kAtomVals == 256, "atom width");

// 16-byte chunk j of row r inside a box: the TMA swizzle (64 or 128 bytes)
// XORs the chunk index with address bits 7..8 or 7..9.
__device__ __forceinline__ int swz(int lane) {
  return kAtomCode == 64 ? (lane >> 1) & 3 : lane & 7;
}
constexpr unsigned long long kLWaitNs = 2000000000ull;

constexpr int kPfxMax = kLanePfxMax;     // per-expert table entries (virtual experts + 1)

// Shared memory: [barriers][pass prefix][cost prefix][tokens][scan scratch],
// then the slots from the next 1024-byte boundary.
template <int NPROJ>
struct LaneCfg {
  static constexpr int D = MOE_LANE_SLOTS;        // slots per warp
  static constexpr int CODE = NPROJ * kBox;       // code bytes per slot
  static constexpr int XB = kAtomVals * (NPROJ == 2 ? 2 : 4);  // token bytes per atom
  static constexpr int SC_OFF = CODE + kRMax * XB;  // scale bytes: [NPROJ][32 rows][kBlk]
  static constexpr int SC = 32 * kBlk;              // scale bytes per projection
  static constexpr int ALIGN = kAtomCode == 64 ? 512 : 1024;  // swizzle span
  static constexpr int SLOT = (SC_OFF + 2 * SC + ALIGN - 1) / ALIGN * ALIGN;
  static constexpr int SLOTS = kLW * D;
  static constexpr int HEAD = SLOTS * 8 + 3 * kPfxMax * 4 + 2 * kLW * 4;
  static constexpr int SMEM = 1024 + HEAD + SLOTS * SLOT;
};
static_assert(LaneCfg<2>::SMEM + 1024 <= 227 * 1024, "shared memory per block");
static_assert(LaneCfg<1>::SMEM + 1024 <= 227 * 1024, "shared memory per block");

struct LaneArgs {
  float* part;    // split-block partial sums: [warp][2][kRMax][NPROJ][32]
  uint32_t* cnt;  // split-block atom counts, one per row block
  int* tab;       // split-block contributors: [row block][NA], slot index + 1
  int NA;         // atoms per row: ceil(K / 256)
  int RB;         // row blocks per projection: ROWS / 32
};

// ------------------------------------------------------------- primitives ---
__device__ __forceinline__ uint32_t lsm(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ unsigned long long lane_now() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ bool lane_try(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Lane 0 waits for the phase (bounded); the outcome is warp-uniform.
__device__ __forceinline__ bool lane_wait(uint32_t bar, uint32_t parity, int* err, int where) {
  int ok = 1;
  if ((threadIdx.x & 31) == 0 && !lane_try(bar, parity)) {
    const unsigned long long t0 = lane_now();
    while (!lane_try(bar, parity)) {
      if (lane_now() - t0 > kLWaitNs) {
        latch_error(err, MOE_ERR_TIMEOUT, where);
        ok = 0;
        break;
      }
    }
  }
  return __shfl_sync(kFull, ok, 0) != 0;
}
__device__ __forceinline__ void lane_tma(uint32_t dst, const CUtensorMap* map, int x, int y,
                                         uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}
// Loads that do not allocate in L1 (scale bytes: each 32-byte sector serves
// eight atoms of one row, L2 keeps it between them).
__device__ __forceinline__ uint32_t ldg_na4(const void* p) {
  uint32_t v;
  asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(v) : "l"(p));
  return v;
}
__device__ __forceinline__ void lane_cp4(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void lane_bulk(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}
__device__ __forceinline__ float2 lane_ffma2(float2 a, float2 b, float2 c) {
  unsigned long long ra, rb, rc, rd;
  ra = (static_cast<unsigned long long>(__float_as_uint(a.y)) << 32) | __float_as_uint(a.x);
  rb = (static_cast<unsigned long long>(__float_as_uint(b.y)) << 32) | __float_as_uint(b.x);
  rc = (static_cast<unsigned long long>(__float_as_uint(c.y)) << 32) | __float_as_uint(c.x);
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(rd) : "l"(ra), "l"(rb), "l"(rc));
  return make_float2(__uint_as_float(uint32_t(rd)), __uint_as_float(uint32_t(rd >> 32)));
}
// scale bytes of a lane's row for one atom: kBlk bytes
using ScaleWord = std::conditional_t<kBlk == 4, uint32_t, uint2>;
__device__ __forceinline__ uint32_t scale_byte(uint32_t s, int j) { return (s >> (8 * j)) & 0xffu; }
__device__ __forceinline__ uint32_t scale_byte(uint2 s, int j) {
  return ((j < 4 ? s.x : s.y) >> (8 * (j & 3))) & 0xffu;
}

// MXFP4 round trip of a 32-value block held one value per lane (OCP MX v1.0
// scale 2^(floor(log2 amax) - 2), RNE onto E2M1, saturating); all lanes call.
__device__ __forceinline__ float mx_round_warp(float v) {
  float amax = fabsf(v);
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, off));
  const int X = mx_scale_exponent(amax);
  const uint32_t byte = f32x2_to_e2m1x2(v * exp2i(-X > 127 ? 127 : -X), 0.f);
  uint32_t h2[4];
  e2m1x8_to_f16x2(byte, h2);
  return f16x2_to_f32x2(h2[0]).x * exp2i(X);
}

// ---------------------------------------------------------- work iterator ---
// Row blocks of the flat space: blk = (pfx[v] + pass) * RB + rb, where pfx[v]
// counts the passes of the virtual experts before v.  A warp walks its atom range [a, A1) segment by
// segment (segment = the part of the range inside one row block).
struct LaneIt {
  int a, seg0, seg1, A1;
  int blk, v, pass, rb;
  bool valid;
};

__device__ __forceinline__ int tokens_of(const FfnArgs& a, int v, int nA) {
  if (v >= nA) return a.T;
  const int e = __ldg(a.plan + 1 + v);
  return __ldg(a.offsets + e + 1) - __ldg(a.offsets + e);
}

// (v, pass) of pass-block vb: the last v with pfx[v] <= vb.
__device__ __forceinline__ void pass_block(const int* pfx, int nV, int vb, int& v, int& pass) {
  int lo = 0, hi = nV - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (pfx[mid] <= vb) lo = mid;
    else hi = mid - 1;
  }
  v = lo;
  pass = vb - pfx[lo];
}

__device__ __forceinline__ void it_segment(LaneIt& it, const LaneArgs& l, const int* pfx,
                                           int nV) {
  if (it.a >= it.A1) {
    it.valid = false;
    return;
  }
  it.blk = it.a / l.NA;
  it.seg0 = it.a;
  it.seg1 = min(it.A1, (it.blk + 1) * l.NA);
  it.rb = it.blk % l.RB;
  pass_block(pfx, nV, it.blk / l.RB, it.v, it.pass);
  it.valid = true;
}
__device__ __forceinline__ void it_begin(LaneIt& it, int A0, int A1, const LaneArgs& l,
                                         const int* pfx, int nV) {
  it.a = A0;
  it.A1 = A1;
  it_segment(it, l, pfx, nV);
}
__device__ __forceinline__ void it_next(LaneIt& it, const LaneArgs& l, const int* pfx, int nV) {
  if (++it.a == it.seg1) it_segment(it, l, pfx, nV);
}

// Cost-balanced split of the flat space over the grid's warps.  Expert v
// costs npass_v + R_v units of RB * NA cost (each pass: one per atom, plus
// one per atom and token); cpfx[v] is the units before v.  Warp g starts at
// the first atom whose start cost is at least g * B, B = ceil(total / NW).
struct LanePart {
  const int* pfx;   // passes before v, [nV + 1]
  const int* cpfx;  // cost units before v, [nV + 1]
  const int* rv;    // tokens of v, [nV]
  int nV, RBNA, B, total;

  __device__ __forceinline__ int atom_at(int g) const {
    const int c = min(total, g * B);
    if (c >= total) return pfx[nV] * RBNA;
    const int cu = c / RBNA;
    int lo = 0, hi = nV - 1;  // last v with cpfx[v] <= cu
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (cpfx[mid] <= cu) lo = mid;
      else hi = mid - 1;
    }
    const int v = lo;
    const int c1 = c - cpfx[v] * RBNA;
    const int np = pfx[v + 1] - pfx[v];
    const int F = RBNA * (1 + kRMax);  // a pass with kRMax tokens
    const int p = np > 1 ? min(np - 1, c1 / F) : 0;
    const int c2 = c1 - p * F;
    const int w = 1 + min(kRMax, rv[v] - p * kRMax);
    return (pfx[v] + p) * RBNA + (c2 + w - 1) / w;
  }
};

// --------------------------------------------------------------- warp state ---
template <int PHASE>
struct LaneWarp {
  static constexpr int NPROJ = PHASE == 0 ? 2 : 1;
  using C = LaneCfg<NPROJ>;
  const FfnArgs* a;
  const LaneArgs* l;
  const CUtensorMap* maps;  // routed projections, then the shared expert's
  unsigned char* codes;     // this warp's D code slots
  uint64_t* full;           // this warp's D barriers
  const int* pfx;           // pass prefix of the virtual experts
  LanePart part;
  int nA, nV, K, ROWS, nb, lane;
  int gw, A0, A1;           // this warp's index in the grid and atom range
  LaneIt nxt;               // next stage to load
  int jc, ji;               // stages consumed / issued (ji counts empty tail slots)
  int jv;                   // stages issued with a copy in flight
  int ev, ee;               // expert id of virtual expert ev (cache)
  int iv, ipass;            // (virtual expert, pass) of the cached token rows below
  int iR;                   // tokens of that pass
  const void* ixsrc;        // lane t < iR: its token's value row (f16 x or f32 h)
  // per segment being loaded: first atom, TMA row, maps, this lane's scale rows
  int iseg, iy;
  const CUtensorMap* imap;
  const uint8_t* isrc[NPROJ];
  int islot;                // ji % D
  // prologue of the down projection: token-row copies deferred until the
  // SwiGLU rows of the previous kernel are complete
  const void* dsrc[C::D];
  uint32_t ddst[C::D], dbytes[C::D], dfb[C::D];
  int cslot;                // jc % D
  uint32_t cpar;            // (jc / D) & 1

  __device__ __forceinline__ int expert(int v) {
    if (v != ev) {
      ev = v;
      ee = v < nA ? __ldg(a->plan + 1 + v) : -1;
    }
    return ee;
  }

  // Per-segment state of the stage loads (nxt entered a new segment).
  __device__ __forceinline__ void refresh() {
    iseg = nxt.seg0;
    const int e = expert(nxt.v);
    const bool sh = e < 0;
    iy = (sh ? 0 : e * ROWS) + nxt.rb * 32;
    imap = maps + (sh ? NPROJ : 0);
    if (nxt.v != iv || nxt.pass != ipass) {
      iv = nxt.v;
      ipass = nxt.pass;
      const VExpert ve = vexpert(*a, PHASE, iv, nA);
      const int t0 = ipass * kRMax;
      iR = min(kRMax, ve.R - t0);
      ixsrc = nullptr;
      if (lane < iR) {
        if constexpr (PHASE == 0)
          ixsrc = a->xh + size_t(token_of(*a, ve, t0 + lane)) * a->H;
        else
          ixsrc = a->h + size_t(out_row(*a, ve, t0 + lane)) * a->I;
      }
    }
    const size_t row = size_t(nxt.rb * 32 + lane);
#pragma unroll
    for (int pj = 0; pj < NPROJ; ++pj) {
      const uint8_t* sbase;
      if (PHASE == 0)
        sbase = sh ? (pj == 0 ? a->sh.gs : a->sh.us) : (pj == 0 ? a->ex.gs : a->ex.us);
      else
        sbase = sh ? a->sh.ds : a->ex.ds;
      if (!sh) sbase += size_t(e) * ROWS * nb;
      isrc[pj] = sbase + row * nb;
    }
  }

  // Load stage ji (if any) into slot ji % D: the code boxes, the atom's values
  // of the pass's tokens, and the rows' scale bytes.  DJ >= 0: a prologue
  // stage (ji == DJ) whose token-row copy is kept for flush_deferred().
  template <int DJ = -1>
  __device__ __forceinline__ void issue() {
    if (nxt.valid) {
      if (nxt.seg0 != iseg) refresh();
      const int atom = nxt.a - nxt.blk * l->NA;
      const int kbase = atom * kAtomVals;
      const bool whole = kbase + kAtomVals <= K;
      const uint32_t xbytes =
          (whole ? uint32_t(kAtomVals) : uint32_t(K - kbase)) * (PHASE == 0 ? 2 : 4);
      const uint32_t fb = lsm(&full[islot]);
      const uint32_t dst = lsm(codes + size_t(islot) * C::SLOT);
      // this slot's previous contents were read through the generic proxy
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      if (lane == 0) {
        asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(fb),
                     "r"(uint32_t(NPROJ * kBox) + uint32_t(iR) * xbytes)
                     : "memory");
#pragma unroll
        for (int pj = 0; pj < NPROJ; ++pj)
          lane_tma(dst + pj * kBox, imap + pj, atom * kAtomCode, iy, fb);
      }
      __syncwarp();
      const void* xsrc =
          lane < iR
              ? static_cast<const unsigned char*>(ixsrc) + size_t(kbase) * (PHASE == 0 ? 2 : 4)
              : nullptr;
      if constexpr (DJ >= 0) {
        dsrc[DJ] = xsrc;
        ddst[DJ] = dst + C::CODE + lane * C::XB;
        dbytes[DJ] = xbytes;
        dfb[DJ] = fb;
      } else if (xsrc != nullptr) {
        lane_bulk(dst + C::CODE + lane * C::XB, xsrc, xbytes, fb);
      }
#pragma unroll
      for (int pj = 0; pj < NPROJ; ++pj) {
        const uint8_t* src = isrc[pj] + atom * kBlk;
        const uint32_t sdst = dst + C::SC_OFF + pj * C::SC + lane * kBlk;
        if (whole) {
#pragma unroll
          for (int w = 0; w < kBlk; w += 4) lane_cp4(sdst + w, src + w);
        } else {  // the last atom of a row: nb - atom * kBlk scale bytes, a multiple of 4
          for (int w = 0; w < nb - atom * kBlk; w += 4) lane_cp4(sdst + w, src + w);
        }
      }
      asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(fb) : "memory");
      it_next(nxt, *l, pfx, nV);
      ++jv;
    }
    else if constexpr (DJ >= 0) {
      dsrc[DJ] = nullptr;
    }
    if (++islot == C::D) islot = 0;
    ++ji;
  }

  // The deferred token-row copies of the prologue stages.
  __device__ __forceinline__ void flush_deferred() {
#pragma unroll
    for (int j = 0; j < C::D; ++j)
      if (dsrc[j] != nullptr) lane_bulk(ddst[j], dsrc[j], dbytes[j], dfb[j]);
  }

  // After a timeout: let the copies already issued land (bounded) so the
  // block's shared memory outlives them.
  __device__ void drain() {
    if (lane == 0) {
      for (int j = jc; j < jv; ++j) {
        const unsigned long long t0 = lane_now();
        while (!lane_try(lsm(&full[j % C::D]), uint32_t(j / C::D) & 1u) &&
               lane_now() - t0 < 100000000ull) {
        }
      }
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
    __syncwarp();
  }

};

// ---------------------------------------------------------- stage compute ---
// Phase 0: gate and up rows of the lane, R tokens (the slot's f16 values).
template <int R>
__device__ __forceinline__ void stage_gateup(const unsigned char* slot, ScaleWord sg, ScaleWord su,
                                             int nblk, int lane, float (&ag)[R], float (&au)[R]) {
  const unsigned char* rg = slot + lane * kAtomCode;
  const unsigned char* ru = slot + kBox + lane * kAtomCode;
  const unsigned char* xs = slot + 2 * kBox;
  const int sw = swz(lane);
#pragma unroll
  for (int j = 0; j < kBlk; ++j) {
    if (kBlk > 4 && j >= nblk) break;
    const uint4 cg = *reinterpret_cast<const uint4*>(rg + ((j ^ sw) << 4));
    const uint4 cu = *reinterpret_cast<const uint4*>(ru + ((j ^ sw) << 4));
    uint32_t wg[16], wu[16];
    e2m1x8_to_f16x2(cg.x, *reinterpret_cast<uint32_t(*)[4]>(&wg[0]));
    e2m1x8_to_f16x2(cg.y, *reinterpret_cast<uint32_t(*)[4]>(&wg[4]));
    e2m1x8_to_f16x2(cg.z, *reinterpret_cast<uint32_t(*)[4]>(&wg[8]));
    e2m1x8_to_f16x2(cg.w, *reinterpret_cast<uint32_t(*)[4]>(&wg[12]));
    e2m1x8_to_f16x2(cu.x, *reinterpret_cast<uint32_t(*)[4]>(&wu[0]));
    e2m1x8_to_f16x2(cu.y, *reinterpret_cast<uint32_t(*)[4]>(&wu[4]));
    e2m1x8_to_f16x2(cu.z, *reinterpret_cast<uint32_t(*)[4]>(&wu[8]));
    e2m1x8_to_f16x2(cu.w, *reinterpret_cast<uint32_t(*)[4]>(&wu[12]));
    const float fg = e8m0_to_f32(scale_byte(sg, j));
    const float fu = e8m0_to_f32(scale_byte(su, j));
#pragma unroll
    for (int t = 0; t < R; ++t) {
      const uint4* xp = reinterpret_cast<const uint4*>(xs + t * (kAtomVals * 2) + j * 64);
      const uint4 x0 = xp[0], x1 = xp[1], x2 = xp[2], x3 = xp[3];
      const uint32_t xv[16] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w,
                               x2.x, x2.y, x2.z, x2.w, x3.x, x3.y, x3.z, x3.w};
      float g0 = 0.f, g1 = 0.f, u0 = 0.f, u1 = 0.f;
#pragma unroll
      for (int p = 0; p < 16; p += 2) {
        g0 = fma2_f16_f32(wg[p], xv[p], g0);
        u0 = fma2_f16_f32(wu[p], xv[p], u0);
        g1 = fma2_f16_f32(wg[p + 1], xv[p + 1], g1);
        u1 = fma2_f16_f32(wu[p + 1], xv[p + 1], u1);
      }
      ag[t] = fmaf(fg, g0 + g1, ag[t]);
      au[t] = fmaf(fu, u0 + u1, au[t]);
    }
  }
}

// Phase 1: down row of the lane, R tokens (the slot's f32 values).
template <int R>
__device__ __forceinline__ void stage_down(const unsigned char* slot, ScaleWord sd, int nblk,
                                           int lane, float (&ad)[R]) {
  const unsigned char* rd = slot + lane * kAtomCode;
  const unsigned char* xs = slot + kBox;
  const int sw = swz(lane);
#pragma unroll
  for (int j = 0; j < kBlk; ++j) {
    if (kBlk > 4 && j >= nblk) break;
    const uint4 c = *reinterpret_cast<const uint4*>(rd + ((j ^ sw) << 4));
    uint32_t w[16];
    e2m1x8_to_f16x2(c.x, *reinterpret_cast<uint32_t(*)[4]>(&w[0]));
    e2m1x8_to_f16x2(c.y, *reinterpret_cast<uint32_t(*)[4]>(&w[4]));
    e2m1x8_to_f16x2(c.z, *reinterpret_cast<uint32_t(*)[4]>(&w[8]));
    e2m1x8_to_f16x2(c.w, *reinterpret_cast<uint32_t(*)[4]>(&w[12]));
    float2 wf[16];
#pragma unroll
    for (int p = 0; p < 16; ++p) wf[p] = f16x2_to_f32x2(w[p]);
    const float fd = e8m0_to_f32(scale_byte(sd, j));
#pragma unroll
    for (int t = 0; t < R; ++t) {
      const float4* xp = reinterpret_cast<const float4*>(xs + t * (kAtomVals * 4) + j * 128);
      float2 s0 = make_float2(0.f, 0.f), s1 = s0, s2 = s0, s3 = s0;
#pragma unroll
      for (int q = 0; q < 8; q += 2) {
        const float4 xa = xp[q], xb = xp[q + 1];
        s0 = lane_ffma2(wf[2 * q], make_float2(xa.x, xa.y), s0);
        s1 = lane_ffma2(wf[2 * q + 1], make_float2(xa.z, xa.w), s1);
        s2 = lane_ffma2(wf[2 * q + 2], make_float2(xb.x, xb.y), s2);
        s3 = lane_ffma2(wf[2 * q + 3], make_float2(xb.z, xb.w), s3);
      }
      ad[t] = fmaf(fd, ((s0.x + s0.y) + (s1.x + s1.y)) + ((s2.x + s2.y) + (s3.x + s3.y)), ad[t]);
    }
  }
}

// Epilogue of one (token row, row) value pair / value.
template <int PHASE>
__device__ __forceinline__ void lane_store(const FfnArgs& a, int orow, int row, float v0,
                                           float v1) {
  if constexpr (PHASE == 0) {
    float hv = v0 / (1.f + expf(-v0)) * v1;
    if (a.act_mxfp4) hv = mx_round_warp(hv);
    a.h[size_t(orow) * a.I + row] = hv;
  } else {
    a.partial[size_t(orow) * a.H + row] = v0;
  }
}

// One segment (one pass of a row block, or the part of it in this warp's
// range): its stages, then its results.  Returns false if a wait timed out.
template <int PHASE, int R>
__device__ bool run_pass(LaneWarp<PHASE>& W, LaneIt& cur, const VExpert& ve) {
  constexpr int NPROJ = LaneWarp<PHASE>::NPROJ;
  using C = LaneCfg<NPROJ>;
  const FfnArgs& a = *W.a;
  const LaneArgs& l = *W.l;
  const int lane = W.lane;
  const int t0 = cur.pass * kRMax;
  const int seg0 = cur.seg0, nst = cur.seg1 - cur.seg0;
  const int blk = cur.blk;
  const int row = cur.rb * 32 + lane;
  int orow[R];
#pragma unroll
  for (int t = 0; t < R; ++t) orow[t] = out_row(a, ve, t0 + t);
  float acc0[R], acc1[R];
#pragma unroll
  for (int t = 0; t < R; ++t) acc0[t] = acc1[t] = 0.f;

  for (int s = 0; s < nst; ++s) {
    const int d = W.cslot;
    const int atom = cur.a - blk * l.NA;
    if (!lane_wait(lsm(&W.full[d]), W.cpar, a.err, 410)) return false;
    const unsigned char* slot = W.codes + size_t(d) * C::SLOT;
    ScaleWord sc[NPROJ];
#pragma unroll
    for (int pj = 0; pj < NPROJ; ++pj)
      sc[pj] = *reinterpret_cast<const ScaleWord*>(slot + C::SC_OFF + pj * C::SC + lane * kBlk);
    const int nblk = min(kBlk, W.nb - atom * kBlk);
    if constexpr (PHASE == 0) {
      stage_gateup<R>(slot, sc[0], sc[1], nblk, lane, acc0, acc1);
    } else {
      stage_down<R>(slot, sc[0], nblk, lane, acc0);
    }
    __syncwarp();
    ++W.jc;
    if (++W.cslot == C::D) {
      W.cslot = 0;
      W.cpar ^= 1u;
    }
    W.issue();
    it_next(cur, l, W.pfx, W.nV);
  }

  const long long B0 = (long long)blk * l.NA;
  if (seg0 == B0 && nst == l.NA) {  // whole row block: final values
#pragma unroll
    for (int t = 0; t < R; ++t) lane_store<PHASE>(a, orow[t], row, acc0[t], acc1[t]);
    return true;
  }
  // split row block: this warp's slot (0 for the first block of its range)
  const int slot_id = W.gw * 2 + (seg0 == W.A0 ? 0 : 1);
  {
    float* slotp = l.part + size_t(slot_id) * (kRMax * NPROJ * 32);
#pragma unroll
    for (int t = 0; t < R; ++t) {
      slotp[(t * NPROJ) * 32 + lane] = acc0[t];
      if constexpr (NPROJ == 2) slotp[(t * NPROJ + 1) * 32 + lane] = acc1[t];
    }
  }
  int* tab = l.tab + size_t(blk) * l.NA;
  if (lane == 0) tab[seg0 - B0] = slot_id + 1;
  __threadfence();
  __syncwarp();
  int last = 0;
  if (lane == 0) last = atomicAdd(l.cnt + blk, uint32_t(nst)) + uint32_t(nst) == uint32_t(l.NA);
  last = __shfl_sync(kFull, last, 0);
  if (!last) return true;
  __threadfence();
  // the contributors' slots in the order of their first atoms
  float sum0[R], sum1[R];
#pragma unroll
  for (int t = 0; t < R; ++t) sum0[t] = sum1[t] = 0.f;
  for (int base = 0; base < l.NA; base += 32) {
    const int id = base + lane < l.NA ? __ldcg(tab + base + lane) : 0;
    if (base + lane < l.NA && id != 0) tab[base + lane] = 0;
    unsigned m = __ballot_sync(kFull, id != 0);
    while (m) {
      const int src = __ffs(m) - 1;
      m &= m - 1;
      const int sid = __shfl_sync(kFull, id, src) - 1;
      const float* sp = l.part + size_t(sid) * (kRMax * NPROJ * 32);
#pragma unroll
      for (int t = 0; t < R; ++t) {
        sum0[t] += __ldcg(sp + (t * NPROJ) * 32 + lane);
        if constexpr (NPROJ == 2) sum1[t] += __ldcg(sp + (t * NPROJ + 1) * 32 + lane);
      }
    }
  }
#pragma unroll
  for (int t = 0; t < R; ++t) lane_store<PHASE>(a, orow[t], row, sum0[t], sum1[t]);
  if (lane == 0) atomicExch(l.cnt + blk, 0u);
  return true;
}

// Tensor maps of the code matrices: the routed experts' projections, then
// the shared expert's (phase 0: gate, up, shared gate, shared up; phase 1:
// down, shared down).
struct LaneMaps {
  CUtensorMap m[4];
};

template <int PHASE>
__global__ void __launch_bounds__(kLThreads, 1)
    k_ffn_lane(const __grid_constant__ FfnArgs a, const __grid_constant__ LaneArgs l,
               const __grid_constant__ LaneMaps maps) {
  constexpr int NPROJ = PHASE == 0 ? 2 : 1;
  using C = LaneCfg<NPROJ>;
  extern __shared__ __align__(16) unsigned char lane_smem[];
  const uint32_t raw = lsm(lane_smem);
  unsigned char* codes = lane_smem + (((raw + C::HEAD + 1023u) & ~1023u) - raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(lane_smem);
  int* s_pfx = reinterpret_cast<int*>(lane_smem + C::SLOTS * 8);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  LaneWarp<PHASE> W;
  W.a = &a;
  W.l = &l;
  W.maps = maps.m;
  W.codes = codes + size_t(warp) * C::D * C::SLOT;
  W.full = bars + warp * C::D;
  if (lane == 0) {
    for (int d = 0; d < C::D; ++d)
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 33;" ::"r"(lsm(&W.full[d])));
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncwarp();
  // The down projection's routing data (plan, buckets) and weights are ready
  // before the previous kernel (gate/up) ends: its setup and first weight
  // loads run ahead of the wait; only its token rows (h) wait.
  if constexpr (PHASE == 0) pdl_wait();
  pdl_trigger();

  W.K = PHASE == 0 ? a.H : a.I;
  W.ROWS = PHASE == 0 ? a.I : a.H;
  W.nb = W.K / 32;
  W.nA = __ldg(a.plan);
  W.nV = W.nA + (a.has_shared ? 1 : 0);
  W.lane = lane;
  W.jc = W.ji = W.jv = 0;
  W.ev = -1;
  W.ee = -1;
  W.iv = -1;
  W.ipass = -1;
  W.iseg = -1;
  W.islot = W.cslot = 0;
  W.cpar = 0;


  // Per virtual expert: tokens, passes and cost; prefix sums over the experts
  // (two entries per thread), or the same tables as the fused router tail
  // wrote them.
  if (a.lane_pre != nullptr) {
    for (int i = threadIdx.x; i <= W.nV; i += blockDim.x) {
      s_pfx[i] = __ldg(a.lane_pre + kPfxMax + i);
      s_pfx[kPfxMax + i] = __ldg(a.lane_pre + 2 * kPfxMax + i);
      s_pfx[2 * kPfxMax + i] = __ldg(a.lane_pre + i);
    }
    __syncthreads();
  } else {
    int* s_cpfx = s_pfx + kPfxMax;
    int* s_rv = s_cpfx + kPfxMax;
    int* s_wsum = s_rv + kPfxMax;  // [kLW][2]
    const int tid = threadIdx.x;
    int np[2] = {0, 0}, cu[2] = {0, 0};
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int v = 2 * tid + i;
      if (v < W.nV) {
        const int R = tokens_of(a, v, W.nA);
        s_rv[v] = R;
        np[i] = (R + kRMax - 1) / kRMax;
        cu[i] = np[i] + R;
      }
    }
    int inp = np[0] + np[1], icu = cu[0] + cu[1];
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int up = __shfl_up_sync(kFull, inp, off), uc = __shfl_up_sync(kFull, icu, off);
      if (lane >= off) {
        inp += up;
        icu += uc;
      }
    }
    if (lane == 31) {
      s_wsum[2 * warp] = inp;
      s_wsum[2 * warp + 1] = icu;
    }
    __syncthreads();
    int bp = 0, bc = 0;
    for (int w = 0; w < warp; ++w) {
      bp += s_wsum[2 * w];
      bc += s_wsum[2 * w + 1];
    }
    int ep = bp + inp - np[0] - np[1], ec = bc + icu - cu[0] - cu[1];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int v = 2 * tid + i;
      if (v <= W.nV) {
        s_pfx[v] = ep;
        s_cpfx[v] = ec;
      }
      ep += np[i];
      ec += cu[i];
    }
    __syncthreads();
  }
  {
    int* s_cpfx = s_pfx + kPfxMax;
    int* s_rv = s_cpfx + kPfxMax;
    W.pfx = s_pfx;
    W.part.pfx = s_pfx;
    W.part.cpfx = s_cpfx;
    W.part.rv = s_rv;
    W.part.nV = W.nV;
    W.part.RBNA = l.RB * l.NA;
    W.part.total = s_cpfx[W.nV] * W.part.RBNA;
    const int NW = gridDim.x * kLW;
    W.part.B = (W.part.total + NW - 1) / NW;
  }

  W.gw = blockIdx.x * kLW + warp;
  W.A0 = W.part.atom_at(W.gw);
  W.A1 = W.part.atom_at(W.gw + 1);
  if (W.A0 >= W.A1) {
    if constexpr (PHASE == 1) pdl_wait();
    return;
  }

  LaneIt cur;
  it_begin(cur, W.A0, W.A1, l, W.pfx, W.nV);
  it_begin(W.nxt, W.A0, W.A1, l, W.pfx, W.nV);
  if constexpr (PHASE == 1) {
    static_assert(C::D <= 4, "prologue");
    W.template issue<0>();
    if constexpr (C::D > 1) W.template issue<1>();
    if constexpr (C::D > 2) W.template issue<2>();
    if constexpr (C::D > 3) W.template issue<3>();
    pdl_wait();
    W.flush_deferred();
  } else {
    for (int d = 0; d < C::D; ++d) W.issue();
  }

  int vv = -1;
  VExpert ve{};
  bool ok = true;
  while (ok && cur.valid) {
    if (cur.v != vv) {
      vv = cur.v;
      ve = vexpert(a, PHASE, vv, W.nA);
    }
    switch (min(kRMax, ve.R - cur.pass * kRMax)) {
      case 1: ok = run_pass<PHASE, 1>(W, cur, ve); break;
      case 2: ok = run_pass<PHASE, 2>(W, cur, ve); break;
      case 3: ok = run_pass<PHASE, 3>(W, cur, ve); break;
      case 4: ok = run_pass<PHASE, 4>(W, cur, ve); break;
      case 5: ok = run_pass<PHASE, 5>(W, cur, ve); break;
      case 6: ok = run_pass<PHASE, 6>(W, cur, ve); break;
      case 7: ok = run_pass<PHASE, 7>(W, cur, ve); break;
      default: ok = run_pass<PHASE, 8>(W, cur, ve); break;
    }
  }
  if (!ok) W.drain();
}

template <int PHASE>
cudaError_t launch_lane_phase(const FfnArgs& a, const LaneArgs& l, const LaneMaps& maps,
                              cudaStream_t st) {
  using C = LaneCfg<PHASE == 0 ? 2 : 1>;
  auto kern = k_ffn_lane<PHASE>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  const int grid = device_info().sm_count < kLaneMaxCtas ? device_info().sm_count : kLaneMaxCtas;
  return launch_pdl(kern, dim3(grid), dim3(kLThreads), size_t(C::SMEM), st, a, l, maps);
}

}  // namespace

bool lane_supported(const moe_shape_t& s) {
  // scale bytes move in 4-byte words (K a multiple of 128 for both phases)
  const int smem = LaneCfg<2>::SMEM > LaneCfg<1>::SMEM ? LaneCfg<2>::SMEM : LaneCfg<1>::SMEM;
  // the per-expert tables hold 256 routed experts and the shared one
  const bool prefix_fits = s.E + 2 <= kPfxMax;
  return s.T <= kLaneMaxT && s.H % 128 == 0 && s.I % 128 == 0 && prefix_fits &&
         device_info().max_smem_optin >= smem;
}

cudaError_t launch_ffn_lane(const FfnArgs& a, float* lane_part, uint32_t* lane_cnt,
                            int* lane_tab, cudaStream_t st) {
  moe_shape_t s{a.T, a.H, a.I, a.E, a.k};
  if (!lane_supported(s) || a.xh == nullptr) return cudaErrorNotSupported;
  LaneMaps g{}, d{};
  const uint64_t HB = uint64_t(a.H) / 2, IB = uint64_t(a.I) / 2;
  bool ok = make_tma_map_u8_box(&g.m[0], a.ex.gq, HB, uint64_t(a.E) * a.I, kAtomCode, 32) &&
            make_tma_map_u8_box(&g.m[1], a.ex.uq, HB, uint64_t(a.E) * a.I, kAtomCode, 32) &&
            make_tma_map_u8_box(&d.m[0], a.ex.dq, IB, uint64_t(a.E) * a.H, kAtomCode, 32);
  if (a.has_shared) {
    ok = ok && make_tma_map_u8_box(&g.m[2], a.sh.gq, HB, a.I, kAtomCode, 32) &&
         make_tma_map_u8_box(&g.m[3], a.sh.uq, HB, a.I, kAtomCode, 32) &&
         make_tma_map_u8_box(&d.m[1], a.sh.dq, IB, a.H, kAtomCode, 32);
  } else {
    g.m[2] = g.m[0];
    g.m[3] = g.m[1];
    d.m[1] = d.m[0];
  }
  if (!ok) return cudaErrorNotSupported;
  LaneArgs l0{lane_part, lane_cnt, lane_tab, (a.H + kAtomVals - 1) / kAtomVals, a.I / 32};
  LaneArgs l1{lane_part, lane_cnt, lane_tab, (a.I + kAtomVals - 1) / kAtomVals, a.H / 32};
  cudaError_t e = launch_lane_phase<0>(a, l0, g, st);
  if (e != cudaSuccess) return e;
  return launch_lane_phase<1>(a, l1, d, st);
}

}  // namespace moe
