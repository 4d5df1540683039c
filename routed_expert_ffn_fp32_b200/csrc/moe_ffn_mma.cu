// Row-block GEMV of the expert FFN for small batches on mma.sync fragments
// (sm_100a).
//
// Computes the two phases of the routed-expert FFN of the MoE layer (per
// routed pair, SwiGLU of the gate/up projections of the token, then the down
// projection) for batches of at most kLaneMaxT tokens, where every expert sees
// only a few rows of activations and the work is a stream of MXFP4 weights
// past a handful of token vectors ("antirez ds4 DeepSeek Metal inference",
// section 技术深度解析: only the activated experts' weights are read; the
// stream of those weights is the cost).
//
// Work decomposition.  A projection's weight matrix [ROWS, K] is cut into
// row blocks of 32 rows and, along K, into atoms of 128 values (64 code bytes
// per row).  The atoms of all (virtual expert, pass, row block) triples form
// one flat index space, atom fastest; every warp of the grid takes a
// contiguous range of it of equal cost (an atom of a pass with R tokens costs
// 1 + R).
//
// Arithmetic.  A warp computes its 32-row block as two 16-row tiles of
// mma.sync.m16n8k16 (f16 inputs, f32 accumulation): the weights are the A
// operand, the pass's tokens the N = 8 columns of B.  Each thread converts one
// 32-bit code word per tile row (8 E2M1 values, cvt.rn.f16x2.e2m1x2) straight
// into the A fragments of two MMAs: within a 32-value scale block thread c of
// a quad owns values 8c..8c+7, so the fragment's k order is a fixed
// permutation of the block that B follows as well (one 16-byte load of a
// token row per block and thread).  The two MMAs of a block start from zero
// and the block's E8M0 scale (decoded by the hardware ue8m0 conversion, so
// byte 0 is 2^-127 and byte 255 NaN) multiplies their sum into the float32
// accumulators: every product is exact (f16 x f16 fits a float32) and the sums
// are float32, though the order of the additions inside an MMA is the
// hardware's, not a scalar loop's.
//
// Operand range.  f16 holds magnitudes up to 65504, so the operands carry
// powers of two: token row t enters as x * 2^-s_t (its largest magnitude in
// [1, 2), s_t written with the f16 rows) and the gate/up sums are
// multiplied by 2^s_t before the SwiGLU; the SwiGLU output h enters the down
// projection as the pair hi = f16(h * 2^-e), lo = f16(h * 2^-e - hi) with one
// exponent e per 32-value block of a row (its largest magnitude in
// [2^14, 2^15)), applied to the block's MMA sums before the weight scale.
// Every bf16 token value within 2^-17 of its row's largest magnitude is exact
// and every h value within 2^-18 of its block's largest magnitude keeps 22
// significant bits.
//
// Data movement.  Each warp keeps D slots of shared memory.  A slot holds the
// 32 x 64-byte code box of an atom per projection, loaded by a TMA tile copy
// (64-byte swizzle: the 4-byte fragment loads of the 32 lanes fall in distinct
// banks), and the atom's 128 f16 values of each operand row (1-D bulk copies,
// one per row; the down projection adds the 16 bytes of block exponents of
// four atoms per token).  Scale bytes come in TMA boxes of 32 rows x 16 bytes
// (four atoms) where a row's scale bytes are a multiple of 16, else one 4-byte
// cp.async per row and atom.  All complete on the slot's mbarrier; the copy
// for stage j + D is issued as soon as stage j has been consumed.  Weight
// loads carry an L2 evict-first policy (read once per call).
//
// Tokens.  A pass handles up to kRMax tokens of an expert; an expert with
// more tokens has one row block per pass in the flat index space (its weights
// are streamed once per pass).
//
// Results.  A warp whose range covers a whole row block writes the block's
// outputs directly (phase 0: SwiGLU as the f16 pair into h; phase 1: the
// expert output row).  A row block split between warps is finished
// deterministically by the warp that holds its first atom (see run_pass).
//
// Every wait is bounded (globaltimer; the limit is a workspace word); on
// expiry the kernel latches MOE_ERR_TIMEOUT, lets its in-flight copies land
// and returns.
#include <cuda.h>

#include "moe_internal.cuh"

namespace moe {

bool make_tma_map_u8_box(CUtensorMap* m, const void* base, uint64_t row_bytes, uint64_t rows,
                         uint32_t box_bytes, uint32_t box_rows);
bool make_tma_map_u8_plain(CUtensorMap* m, const void* base, uint64_t row_bytes, uint64_t rows,
                           uint32_t box_bytes, uint32_t box_rows);

namespace {

constexpr int kRMax = kLaneRMax;         // tokens per pass
static_assert(kRMax == 8, "a pass fills the eight MMA columns (gate/up)");
constexpr int kAtomVals = 128;           // K values of a row per atom
constexpr int kAtomCode = kAtomVals / 2; // code bytes of a row per atom
constexpr int kBlk = kAtomVals / 32;     // scale blocks per atom
constexpr int kBox = 32 * kAtomCode;     // one projection's 32-row code box
constexpr int kXRow = kAtomVals * 2;     // one f16 operand row of an atom
constexpr int kXExp = 16;                // block exponents of one h row, four atoms
constexpr int kPfxMax = kLanePfxMax;     // per-expert table entries (virtual experts + 1)
constexpr int kEntMax = 512;             // bucket entries staged in shared memory
constexpr int kOwnMax = 32;              // contributors listed per split block
constexpr int kSlotF = kRMax * 2 * 32;   // floats of one split-block slot

// Shared memory: [barriers][pass prefix][cost prefix][tokens][plan][offsets]
// [scan scratch][entries][contributor lists][token exponents], then from the
// next 1024-byte boundary per warp its D stage slots (code boxes, operand
// rows), its NSCE scale entries and (down) its D block-exponent chunks.
// A scale entry holds [NPROJ][32 rows][16 bytes]: the scale bytes of four
// atoms of each row (one TMA box per projection), or of one atom (cp.async)
// when a row's scale bytes are not a multiple of 16.
template <int NPROJ>
struct LaneCfg {
  static constexpr int NW = kLaneWarps;            // warps per CTA
  static constexpr int THREADS = 32 * NW;
  static constexpr int D = 3;                      // slots per warp
  static constexpr int CODE = NPROJ * kBox;                     // code bytes per slot
  static constexpr int XROWS = NPROJ == 2 ? kRMax : 2 * kRMax;  // f16 operand rows
  static constexpr int SLOT = CODE + XROWS * kXRow;
  static constexpr int SCE = NPROJ * 32 * 16;                   // one scale entry
  static constexpr int NSCE = 3;                                // scale entries per warp
  static constexpr int EXPB = NPROJ == 1 ? D * kRMax * kXExp : 0;
  static constexpr int WARP_BYTES = (D * SLOT + NSCE * SCE + EXPB + 511) / 512 * 512;
  static constexpr int SLOTS = NW * D;
  static constexpr int HEAD = SLOTS * 8 + 5 * kPfxMax * 4 + 2 * NW * 4 + kEntMax * 4 +
                              NW * kOwnMax * 4 + kLaneMaxT;
  static constexpr int SMEM = 1024 + HEAD + NW * WARP_BYTES;
  static_assert(SLOT % 512 == 0 && SCE % 512 == 0, "64-byte swizzle boxes start on 512 bytes");
  static_assert(D <= NSCE, "a scale entry outlives the stages in flight");
  static_assert(2 * kRMax <= 16, "operand-row copies use lanes below 16");
};
static_assert(LaneCfg<2>::SMEM + 1024 <= 227 * 1024, "shared memory per block");
static_assert(LaneCfg<1>::SMEM + 1024 <= 227 * 1024, "shared memory per block");

struct LaneArgs {
  float* part;    // split-block partial sums, one slot per warp: [grid warp][kSlotF]
  uint32_t* cnt;  // split-block atom counts of the contributors, one per row block, zero at the
                  // call's start
  int NA;         // atoms per row: K / 128
  int RB;         // row blocks per projection: ROWS / 32
  int sbox;       // scale bytes by TMA boxes of 4 atoms (K / 32 a multiple of 16)
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
// Lane 0 waits for the phase (bounded by limit_ns); the outcome is warp-uniform.
__device__ __forceinline__ bool lane_wait(uint32_t bar, uint32_t parity, int* err, int where,
                                          unsigned long long limit_ns) {
  int ok = 1;
  if ((threadIdx.x & 31) == 0 && !lane_try(bar, parity)) {
    const unsigned long long t0 = lane_now();
    while (!lane_try(bar, parity)) {
      if (lane_now() - t0 > limit_ns) {
        latch_error(err, MOE_ERR_TIMEOUT, where);
        ok = 0;
        break;
      }
    }
  }
  return __shfl_sync(kFull, ok, 0) != 0;
}
// TMA tile copy with an L2 cache policy (weights: read once, evict first, so
// the stream does not push out the instructions and the small hot data).
__device__ __forceinline__ void lane_tma_hint(uint32_t dst, const CUtensorMap* map, int x, int y,
                                              uint32_t bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar), "l"(policy)
      : "memory");
}
__device__ __forceinline__ uint64_t evict_first_policy() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
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
// d += A B for one m16n8k16 tile, f16 inputs, f32 accumulators.
__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Four E8M0 bytes (the blocks of one atom of one row, or four biased block
// exponents) as bf16 powers of two: bytes 0, 1 in lo, bytes 2, 3 in hi.
struct Pow4 {
  uint32_t lo, hi;
};
__device__ __forceinline__ Pow4 pow4_of(uint32_t w) {
  return {ue8m0x2_to_bf16x2(w), ue8m0x2_to_bf16x2(w >> 16)};
}
template <int J>
__device__ __forceinline__ float pow_at(const Pow4& p) {
  const uint32_t v = J < 2 ? p.lo : p.hi;
  return __uint_as_float((J & 1) ? (v & 0xffff0000u) : (v << 16));
}

// MXFP4 round trip of v with the block scale exponent X (OCP MX v1.0: RNE
// onto the E2M1 grid, saturating).
__device__ __forceinline__ float mx_round(float v, int X) {
  const uint32_t byte = f32x2_to_e2m1x2(v * exp2i(-X > 127 ? 127 : -X), 0.f);
  uint32_t h2[4];
  e2m1x8_to_f16x2(byte, h2);
  return f16x2_to_f32x2(h2[0]).x * exp2i(X);
}

// Exponent e of the power of two that brings a 32-value block of h with
// largest magnitude amax into [2^14, 2^15) for its f16 pair: clamped to
// [-126, 113]; 0 for a zero or non-finite block.
__device__ __forceinline__ int h_block_exponent(float amax) {
  const uint32_t bits = __float_as_uint(amax);
  if (bits == 0u || bits >= 0x7f800000u) return 0;
  const int field = int(bits >> 23);
  const int e = field == 0 ? -126 : field - 127 - 14;
  return e < -126 ? -126 : e;
}

// ------------------------------------------------------ fragment mapping ---
// Thread (g = lane / 4, c = lane % 4) of an m16n8k16 accumulator holds, for
// row tile mt, element i of
//   rows  mt*16 + g (i = 0, 1) and mt*16 + g + 8 (i = 2, 3),
//   column 2c + (i & 1).
// Phase 0: column = token of the pass.  Phase 1: column 2u + q of column tile
// nt = token nt*4 + u, piece q (0: hi, 1: lo of h).
__device__ __forceinline__ int frag_row(int g, int mt, int i) { return mt * 16 + (i >> 1) * 8 + g; }

// ------------------------------------------------------- routing metadata ---
// The routing arrays every lookup of the kernel needs, preloaded into shared
// memory in one round of independent loads: plan (active experts), offsets
// (bucket starts), the token rows' scale exponents and, for batches of at
// most kEntMax pairs, the bucket entries themselves (larger batches read them
// from global memory).
struct Meta {
  const int* plan;     // [0] active experts nA, [1 + v] expert id of virtual expert v
  const int* off;      // bucket offsets [E + 1]
  const int* ent;      // bucket entries (pair indices), shared or global memory
  const int* rv;       // tokens of virtual expert v
  const uint8_t* xe;   // s_t + 127 of token t
  int nA, nV, T, k;
  __device__ __forceinline__ int expert(int v) const { return v < nA ? plan[1 + v] : -1; }
  // output row (pair index, or T*k + r for the shared expert) of bucket row r
  __device__ __forceinline__ int out_row(int v, int r) const {
    return v < nA ? ent[off[plan[1 + v]] + r] : T * k + r;
  }
  __device__ __forceinline__ int token(int v, int r) const {
    return v < nA ? ent[off[plan[1 + v]] + r] / k : r;
  }
};

// ---------------------------------------------------------- work iterator ---
// Row blocks of the flat space: blk = (pfx[v] + pass) * RB + rb, where pfx[v]
// counts the passes of the virtual experts before v.  A warp walks its atom
// range [a, A1) segment by segment (segment = the part of the range inside
// one row block).
struct LaneIt {
  int a, seg0, seg1, A1;
  int blk, v, pass, rb;
  bool valid;
};

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

  __device__ __forceinline__ void init(const int* p, const int* c, const int* r, int n, int rbna,
                                       int nwarps) {
    pfx = p;
    cpfx = c;
    rv = r;
    nV = n;
    RBNA = rbna;
    total = c[n] * rbna;
    B = (total + nwarps - 1) / nwarps;
  }
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
  const Meta* m;
  const CUtensorMap* maps;  // code maps: routed projections, then the shared expert's
  const CUtensorMap* smaps; // scale maps, same order (TMA scale boxes)
  unsigned char* codes;     // this warp's D code slots
  unsigned char* scales;    // this warp's NSCE scale entries
  unsigned char* exps;      // (down) this warp's D block-exponent chunks [D][kRMax][16]
  int ri;                   // scale entry of the last TMA scale load
  uint32_t sring;           // scale entry of the stage in slot d: bits 2d, 2d + 1
  uint64_t* full;           // this warp's D barriers
  const int* pfx;           // pass prefix of the virtual experts
  LanePart part;
  int nV, K, ROWS, nb, lane;
  int gw;                   // this warp's index in the grid
  unsigned long long wait_ns;
  bool starve;              // debug: stage 0 gets no copies (its wait runs out)
  LaneIt nxt;               // next stage to load
  int jc, ji;               // stages consumed / issued (ji counts empty tail slots)
  uint32_t pend, ppar;      // slots with copies in flight, and their phase parities
  int iv, ipass;            // (virtual expert, pass) of the cached operand rows below
  int irows;                // f16 operand rows of that pass (tokens, or tokens x 2)
  const unsigned char* ixsrc;  // lane < irows: the start of its operand row
  const unsigned char* iesrc;  // (down) lane 16 + t < 16 + tokens: token t's block exponents
  // per segment being loaded: first atom, TMA row, maps, this lane's scale rows
  int iseg, iy;
  const CUtensorMap* imap;
  const CUtensorMap* ismap;
  const uint8_t* isrc[NPROJ];
  int islot;                // ji % D
  // prologue of the down projection: operand copies deferred until the
  // SwiGLU rows of the previous kernel are complete
  const void* dsrc[C::D];
  uint32_t ddst[C::D], dfb[C::D], dsz[C::D];
  int cslot;                // jc % D
  uint32_t cpar;            // (jc / D) & 1
  // the other contributors of the split row block this warp owns at the end
  // of its range (their warp indices, in atom order, in shared memory); on =
  // -1: not listed (none, or more than kOwnMax)
  int* osid;
  int on;

  // Per-segment state of the stage loads (nxt entered a new segment).
  __device__ __forceinline__ void refresh() {
    iseg = nxt.seg0;
    const int e = m->expert(nxt.v);
    const bool sh = e < 0;
    iy = (sh ? 0 : e * ROWS) + nxt.rb * 32;
    imap = maps + (sh ? NPROJ : 0);
    ismap = smaps + (sh ? NPROJ : 0);
    if (nxt.v != iv || nxt.pass != ipass) {
      iv = nxt.v;
      ipass = nxt.pass;
      const int t0 = ipass * kRMax;
      const int R = min(kRMax, m->rv[iv] - t0);
      ixsrc = nullptr;
      iesrc = nullptr;
      if constexpr (PHASE == 0) {
        irows = R;
        if (lane < R)
          ixsrc = reinterpret_cast<const unsigned char*>(a->xh + size_t(m->token(iv, t0 + lane)) * a->H);
      } else {
        // h row of a pair: I f16 values hi, I f16 values lo, block exponents
        irows = 2 * R;
        const size_t pitch = h_pitch(size_t(a->I));
        const unsigned char* hb = reinterpret_cast<const unsigned char*>(a->h);
        if (lane < 2 * R)
          ixsrc = hb + size_t(m->out_row(iv, t0 + (lane >> 1))) * pitch +
                  size_t(lane & 1) * (size_t(a->I) * 2);
        if (lane >= 16 && lane < 16 + R)
          iesrc = hb + size_t(m->out_row(iv, t0 + lane - 16)) * pitch + size_t(a->I) * 4;
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
  // of the pass's operand rows (down: and their block exponents), and the
  // rows' scale bytes.  DJ >= 0: a prologue stage (ji == DJ) whose operand
  // copies are kept for flush_deferred().
  template <int DJ = -1>
  __device__ __forceinline__ void issue() {
    if (nxt.valid) {
      if (nxt.seg0 != iseg) refresh();
      const int atom = nxt.a - nxt.blk * l->NA;
      const int kbase = atom * kAtomVals;
      const uint32_t fb = lsm(&full[islot]);
      const uint32_t dst = lsm(codes + size_t(islot) * C::SLOT);
      // scale entry of this stage: a new TMA box of four atoms at the start
      // of a segment or of a group of four atoms; else the slot's own entry
      bool sload = false;
      int ent = islot;
      if (l->sbox) {
        if (nxt.a == nxt.seg0 || (atom & 3) == 0) {
          ri = ri == C::NSCE - 1 ? 0 : ri + 1;
          sload = true;
        }
        ent = ri;
      }
      sring = (sring & ~(3u << (2 * islot))) | (uint32_t(ent) << (2 * islot));
      const bool skip = starve && ji == 0;
      if (!skip) {
        const uint32_t sdst = lsm(scales + size_t(ent) * C::SCE);
        // this slot's previous contents were read through the generic proxy
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        if (lane == 0) {
          const uint32_t ebytes = PHASE == 1 ? uint32_t(irows / 2) * kXExp : 0u;
          asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(fb),
                       "r"(uint32_t(NPROJ * kBox) + uint32_t(irows) * kXRow + ebytes +
                           (sload ? uint32_t(C::SCE) : 0u))
                       : "memory");
          const uint64_t pol = evict_first_policy();
#pragma unroll
          for (int pj = 0; pj < NPROJ; ++pj)
            lane_tma_hint(dst + pj * kBox, imap + pj, atom * kAtomCode, iy, fb, pol);
          if (sload)
#pragma unroll
            for (int pj = 0; pj < NPROJ; ++pj)
              lane_tma_hint(sdst + pj * (C::SCE / NPROJ), ismap + pj, 16 * (atom >> 2), iy, fb,
                            pol);
        }
        __syncwarp();
        // operand copy of this lane: an operand row, or (down) a token's
        // block exponents of this group of four atoms
        const void* xsrc = nullptr;
        uint32_t xdst = 0, xsz = 0;
        if (ixsrc != nullptr) {
          xsrc = ixsrc + size_t(kbase) * 2;
          xdst = dst + C::CODE + lane * kXRow;
          xsz = kXRow;
        } else if (PHASE == 1 && iesrc != nullptr) {
          xsrc = iesrc + size_t(atom >> 2) * kXExp;
          xdst = lsm(exps + size_t(islot) * (kRMax * kXExp) + (lane - 16) * kXExp);
          xsz = kXExp;
        }
        if constexpr (DJ >= 0) {
          dsrc[DJ] = xsrc;
          ddst[DJ] = xdst;
          dsz[DJ] = xsz;
          dfb[DJ] = fb;
        } else if (xsrc != nullptr) {
          lane_bulk(xdst, xsrc, xsz, fb);
        }
        if (!l->sbox) {
#pragma unroll
          for (int pj = 0; pj < NPROJ; ++pj)
            lane_cp4(sdst + pj * (C::SCE / NPROJ) + lane * 16, isrc[pj] + atom * kBlk);
          asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(fb) : "memory");
        }
        pend |= 1u << islot;
        ppar = (ppar & ~(1u << islot)) | (((uint32_t(ji) / C::D) & 1u) << islot);
      } else if constexpr (DJ >= 0) {
        dsrc[DJ] = nullptr;
      }
      it_next(nxt, *l, pfx, nV);
    } else if constexpr (DJ >= 0) {
      dsrc[DJ] = nullptr;
    }
    if (++islot == C::D) islot = 0;
    ++ji;
  }

  // The deferred operand copies of the prologue stages.
  __device__ __forceinline__ void flush_deferred() {
#pragma unroll
    for (int j = 0; j < C::D; ++j)
      if (dsrc[j] != nullptr) lane_bulk(ddst[j], dsrc[j], dsz[j], dfb[j]);
  }

  // After a timeout: let the copies already issued land (bounded) so the
  // block's shared memory outlives them.
  __device__ void drain() {
    if (lane == 0) {
      for (int d = 0; d < C::D; ++d) {
        if (!((pend >> d) & 1u)) continue;
        const unsigned long long t0 = lane_now();
        while (!lane_try(lsm(&full[d]), (ppar >> d) & 1u) && lane_now() - t0 < 100000000ull) {
        }
      }
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
    __syncwarp();
  }
};

// ---------------------------------------------------------- stage compute ---
// Per-thread byte offsets of the fragment words: row g of a tile, word c of
// scale block j, inside the 64-byte-swizzled box (16-byte chunk j of row r is
// stored at chunk j ^ ((r >> 1) & 3); rows g, g + 8, g + 16, g + 24 share it).
struct FragOfs {
  int w[kBlk];  // code word of row g, block j
  int x;        // operand row g, this thread's 8 values of block 0
  int s;        // scale word of row g in a scale entry (16-byte rows)
};
__device__ __forceinline__ FragOfs frag_ofs(int lane) {
  const int g = lane >> 2, c = lane & 3;
  FragOfs f;
#pragma unroll
  for (int j = 0; j < kBlk; ++j) f.w[j] = g * kAtomCode + ((j ^ ((g >> 1) & 3)) << 4) + 4 * c;
  f.x = g * kXRow + 16 * c;
  f.s = g * 16;
  return f;
}

// One 16-row tile x one 32-value block: the A fragments of its two MMAs from
// the code words of rows g and g + 8, then d = A B with B the block's operand
// values (b: 4 f16x2 registers).
__device__ __forceinline__ void tile_block(const unsigned char* box, int wofs, const uint4& b,
                                           float (&d)[4]) {
  const uint32_t w0 = *reinterpret_cast<const uint32_t*>(box + wofs);
  const uint32_t w1 = *reinterpret_cast<const uint32_t*>(box + wofs + 8 * kAtomCode);
  uint32_t h0[4], h1[4];
  e2m1x8_to_f16x2(w0, h0);
  e2m1x8_to_f16x2(w1, h1);
  d[0] = d[1] = d[2] = d[3] = 0.f;
  mma16816(d, h0[0], h1[0], h0[1], h1[1], b.x, b.y);
  mma16816(d, h0[2], h1[2], h0[3], h1[3], b.z, b.w);
}

// acc (rows g, g + 8 of a tile) += d * (f0, f1).
__device__ __forceinline__ void scale_acc(float (&acc)[4], const float (&d)[4], float f0,
                                          float f1) {
  acc[0] = fmaf(d[0], f0, acc[0]);
  acc[1] = fmaf(d[1], f0, acc[1]);
  acc[2] = fmaf(d[2], f1, acc[2]);
  acc[3] = fmaf(d[3], f1, acc[3]);
}

// Phase 0: gate (p = 0) and up (p = 1) of the block's 32 rows for the pass's
// tokens (the slot's f16 token rows).
template <int J>
__device__ __forceinline__ void gateup_block(const unsigned char* slot, const FragOfs& f,
                                             const Pow4 (&sw)[2][2][2], float (&acc)[2][2][4]) {
  using C = LaneCfg<2>;
  const uint4 b = *reinterpret_cast<const uint4*>(slot + C::CODE + f.x + 64 * J);
#pragma unroll
  for (int p = 0; p < 2; ++p)
#pragma unroll
    for (int mt = 0; mt < 2; ++mt) {
      float d[4];
      tile_block(slot + p * kBox + mt * 16 * kAtomCode, f.w[J], b, d);
      scale_acc(acc[p][mt], d, pow_at<J>(sw[p][mt][0]), pow_at<J>(sw[p][mt][1]));
    }
}
// sc: the stage's scale words in its scale entry ([projection][32 rows][16 B]).
__device__ __forceinline__ void stage_gateup(const unsigned char* slot, const unsigned char* sc,
                                             const FragOfs& f, float (&acc)[2][2][4]) {
  Pow4 sw[2][2][2];  // scales: [projection][tile][row g / g + 8]
#pragma unroll
  for (int p = 0; p < 2; ++p)
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int hh = 0; hh < 2; ++hh)
        sw[p][mt][hh] =
            pow4_of(*reinterpret_cast<const uint32_t*>(sc + p * 512 + f.s + (mt * 16 + hh * 8) * 16));
  gateup_block<0>(slot, f, sw, acc);
  gateup_block<1>(slot, f, sw, acc);
  gateup_block<2>(slot, f, sw, acc);
  gateup_block<3>(slot, f, sw, acc);
}

// Phase 1: down rows for NT column tiles of (token, hi/lo) operand rows; the
// weight scale of a block times the token's block exponent of h.
template <int J, int NT>
__device__ __forceinline__ void down_block(const unsigned char* slot, const FragOfs& f,
                                           const Pow4 (&sw)[2][2], const Pow4 (&ew)[NT],
                                           float (&acc)[NT][2][4]) {
  using C = LaneCfg<1>;
  uint4 b[NT];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
    b[nt] = *reinterpret_cast<const uint4*>(slot + C::CODE + f.x + nt * 8 * kXRow + 64 * J);
#pragma unroll
  for (int mt = 0; mt < 2; ++mt) {
    const unsigned char* box = slot + mt * 16 * kAtomCode;
    const uint32_t w0 = *reinterpret_cast<const uint32_t*>(box + f.w[J]);
    const uint32_t w1 = *reinterpret_cast<const uint32_t*>(box + f.w[J] + 8 * kAtomCode);
    uint32_t h0[4], h1[4];
    e2m1x8_to_f16x2(w0, h0);
    e2m1x8_to_f16x2(w1, h1);
    const float f0 = pow_at<J>(sw[mt][0]), f1 = pow_at<J>(sw[mt][1]);
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      float d[4] = {0.f, 0.f, 0.f, 0.f};
      mma16816(d, h0[0], h1[0], h0[1], h1[1], b[nt].x, b[nt].y);
      mma16816(d, h0[2], h1[2], h0[3], h1[3], b[nt].z, b[nt].w);
      // the block exponent of h first, then the weight scale: each product
      // overflows only where the unscaled term would
      const float fe = pow_at<J>(ew[nt]);
#pragma unroll
      for (int i = 0; i < 4; ++i) d[i] *= fe;
      scale_acc(acc[nt][mt], d, f0, f1);
    }
  }
}
// ex: the stage's block-exponent chunks [kRMax tokens][16 bytes]; atom & 3
// selects the atom's four bytes.
template <int NT>
__device__ __forceinline__ void stage_down(const unsigned char* slot, const unsigned char* sc,
                                           const unsigned char* ex, int atom, const FragOfs& f,
                                           int c, float (&acc)[NT][2][4]) {
  Pow4 sw[2][2];
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int hh = 0; hh < 2; ++hh)
      sw[mt][hh] = pow4_of(*reinterpret_cast<const uint32_t*>(sc + f.s + (mt * 16 + hh * 8) * 16));
  Pow4 ew[NT];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
    ew[nt] = pow4_of(*reinterpret_cast<const uint32_t*>(ex + (nt * 4 + c) * kXExp + 4 * (atom & 3)));
  down_block<0, NT>(slot, f, sw, ew, acc);
  down_block<1, NT>(slot, f, sw, ew, acc);
  down_block<2, NT>(slot, f, sw, ew, acc);
  down_block<3, NT>(slot, f, sw, ew, acc);
}

// ---------------------------------------------------------------- results ---
// Values of a finished row block in fragment order: phase 0 [gate, up][tile]
// [element], phase 1 [column tile][tile][row g / g + 8] (hi + lo summed).
template <int PHASE, int NT>
struct BlockVals {
  static constexpr int N = PHASE == 0 ? 16 : NT * 4;
  float v[N];
};

// Token (of the pass) and row (in the block) of value n, and its slot entry.
template <int PHASE>
__device__ __forceinline__ void val_pos(int n, int g, int c, int& t, int& row, int& proj) {
  if constexpr (PHASE == 0) {
    proj = n >> 3;
    const int mt = (n >> 2) & 1, i = n & 3;
    t = 2 * c + (i & 1);
    row = frag_row(g, mt, i);
  } else {
    proj = 0;
    const int nt = n >> 2, mt = (n >> 1) & 1, hh = n & 1;
    t = nt * 4 + c;
    row = mt * 16 + hh * 8 + g;
  }
}

template <int PHASE, int NT>
__device__ __forceinline__ void collect(const float (&acc)[PHASE == 0 ? 2 : NT][2][4],
                                        BlockVals<PHASE, NT>& o) {
  if constexpr (PHASE == 0) {
#pragma unroll
    for (int p = 0; p < 2; ++p)
#pragma unroll
      for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int i = 0; i < 4; ++i) o.v[p * 8 + mt * 4 + i] = acc[p][mt][i];
  } else {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh)
          o.v[nt * 4 + mt * 2 + hh] = acc[nt][mt][2 * hh] + acc[nt][mt][2 * hh + 1];
  }
}

// Epilogue of a finished row block of virtual expert v, pass tokens t0 ..
// t0 + R - 1 (all lanes call: the block exponent of h reduces over the
// block's 32 rows with shuffles).
template <int PHASE, int NT>
__device__ __forceinline__ void block_store(const FfnArgs& a, const Meta& m, int v, int t0, int R,
                                            int rb, int lane, const BlockVals<PHASE, NT>& o) {
  const int g = lane >> 2, c = lane & 3;
  const int row0 = rb * 32;
  if constexpr (PHASE == 0) {
    // the gate/up sums of tokens 2c and 2c + 1 back to the token rows' scale,
    // then h: [tile][element]
    float sx[2];
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const int t = 2 * c + q;
      sx[q] = t < R ? __uint_as_float(uint32_t(m.xe[m.token(v, t0 + t)]) << 23) : 1.f;
    }
    float hv[8];
#pragma unroll
    for (int n = 0; n < 8; ++n) {
      const float gt = o.v[n] * sx[n & 1], up = o.v[8 + n] * sx[n & 1];
      hv[n] = gt / (1.f + expf(-gt)) * up;
    }
    const size_t pitch = h_pitch(size_t(a.I));
    unsigned char* hbase = reinterpret_cast<unsigned char*>(a.h);
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      // one 32-value block along I per token: the 32 rows of this block,
      // held by the eight threads of quad column c
      float amax = fmaxf(fmaxf(fabsf(hv[q]), fabsf(hv[2 + q])), fmaxf(fabsf(hv[4 + q]), fabsf(hv[6 + q])));
#pragma unroll
      for (int off = 4; off <= 16; off <<= 1) amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, off));
      if (a.act_mxfp4) {
        const int X = mx_scale_exponent(amax);
#pragma unroll
        for (int n = q; n < 8; n += 2) hv[n] = mx_round(hv[n], X);
      }
      const int eb = h_block_exponent(amax);
      const float inv = exp2i(-eb);
      const int t = 2 * c + q;
      if (t < R) {
        unsigned char* hr = hbase + size_t(m.out_row(v, t0 + t)) * pitch;
        uint16_t* hi16 = reinterpret_cast<uint16_t*>(hr);
#pragma unroll
        for (int n = q; n < 8; n += 2) {
          const float hs = hv[n] * inv;
          const __half hi = __float2half_rn(hs);
          const __half lo = __float2half_rn(hs - __half2float(hi));
          const int row = row0 + frag_row(g, n >> 2, n & 3);
          hi16[row] = __half_as_ushort(hi);
          hi16[a.I + row] = __half_as_ushort(lo);
        }
        if (g == 0) hr[size_t(a.I) * 4 + rb] = uint8_t(eb + 127);
      }
    }
  } else {
#pragma unroll
    for (int n = 0; n < NT * 4; ++n) {
      int t, row, p;
      val_pos<1>(n, g, c, t, row, p);
      if (t < R) a.partial[size_t(m.out_row(v, t0 + t)) * a.H + row0 + row] = o.v[n];
    }
  }
}

// One segment (one pass of a row block, or the part of it in this warp's
// range): its stages, then its results.  Returns false if a wait timed out.
//
// A row block split between warps is owned by the warp whose range holds its
// first atom; for that warp it is the last segment of its range, for every
// other contributor the first.  A contributor stores its partial sums in its
// slot and adds its atom count to the block's counter, early in its range and
// without waiting.  The owner, at the end of its range, waits (bounded) until
// the count is complete, adds the contributors' slots after its own sums in
// atom order (the same order whichever warps share the block) and applies the
// epilogue; it then clears the counter.
template <int PHASE, int NT>
__device__ bool run_pass(LaneWarp<PHASE>& W, LaneIt& cur, const FragOfs& f) {
  constexpr int NPROJ = LaneWarp<PHASE>::NPROJ;
  using C = LaneCfg<NPROJ>;
  const FfnArgs& a = *W.a;
  const LaneArgs& l = *W.l;
  const Meta& m = *W.m;
  const int lane = W.lane, g = lane >> 2, c = lane & 3;
  const int v = cur.v, pass = cur.pass, rb = cur.rb;
  const int t0 = pass * kRMax;
  const int R = min(kRMax, m.rv[v] - t0);
  const int seg0 = cur.seg0, nst = cur.seg1 - cur.seg0;
  const int blk = cur.blk;
  float acc[PHASE == 0 ? 2 : NT][2][4];
#pragma unroll
  for (int p = 0; p < (PHASE == 0 ? 2 : NT); ++p)
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[p][mt][i] = 0.f;

  for (int s = 0; s < nst; ++s) {
    const int d = W.cslot;
    if (!lane_wait(lsm(&W.full[d]), W.cpar, a.err, 410, W.wait_ns)) return false;
    const unsigned char* slot = W.codes + size_t(d) * C::SLOT;
    const int atom = cur.a - blk * l.NA;
    const unsigned char* sc = W.scales + size_t((W.sring >> (2 * d)) & 3u) * C::SCE +
                              (l.sbox ? 4 * (atom & 3) : 0);
    if constexpr (PHASE == 0) stage_gateup(slot, sc, f, acc);
    else stage_down<NT>(slot, sc, W.exps + size_t(d) * (kRMax * kXExp), atom, f, c, acc);
    __syncwarp();
    W.pend &= ~(1u << d);
    ++W.jc;
    if (++W.cslot == C::D) {
      W.cslot = 0;
      W.cpar ^= 1u;
    }
    W.issue();
    it_next(cur, l, W.pfx, W.nV);
  }

  BlockVals<PHASE, NT> o;
  collect<PHASE, NT>(acc, o);
  constexpr int NV = BlockVals<PHASE, NT>::N;
  const int B0 = blk * l.NA;
  if (seg0 == B0 && nst == l.NA) {  // whole row block: final values
    block_store<PHASE, NT>(a, m, v, t0, R, rb, lane, o);
    return true;
  }
  if (seg0 != B0) {
    // contributor: partial sums into this warp's slot, then count them in
    float* slotp = l.part + size_t(W.gw) * kSlotF;
#pragma unroll
    for (int n = 0; n < NV; ++n) {
      int t, row, p;
      val_pos<PHASE>(n, g, c, t, row, p);
      if (t < R) slotp[(t * NPROJ + p) * 32 + row] = o.v[n];
    }
    // Count in with a release-ordered add from lane 31: it issues no copies
    // (the operand rows and block exponents take lanes below 24, the tensor
    // copies lane 0), so its release waits only for the slot stores, which
    // __syncwarp orders before it, and not for this warp's stage loads in
    // flight (a full sequentially consistent fence would).
    __syncwarp();
    if (lane == 31)
      asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(l.cnt + blk), "r"(uint32_t(nst))
                   : "memory");
    return true;
  }
  // owner: wait for the other contributors' atoms
  const uint32_t want = uint32_t(l.NA - nst);
  int ok = 1;
  if (lane == 0) {
    uint32_t got;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(got) : "l"(l.cnt + blk) : "memory");
    if (got != want) {
      const unsigned long long t_0 = lane_now();
      do {
        asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(got) : "l"(l.cnt + blk) : "memory");
        if (got != want && lane_now() - t_0 > W.wait_ns) {
          latch_error(a.err, MOE_ERR_TIMEOUT, 420);
          ok = 0;
          break;
        }
      } while (got != want);
    }
  }
  if (!__shfl_sync(kFull, ok, 0)) return false;
  if (W.on >= 0) {
    // the contributors listed at set-up: four slots in flight at a time
    for (int q0 = 0; q0 < W.on; q0 += 4) {
      float val[4][NV];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const bool use = q0 + q < W.on;
        const float* sp = l.part + size_t(use ? W.osid[q0 + q] : 0) * kSlotF;
#pragma unroll
        for (int n = 0; n < NV; ++n) {
          int t, row, p;
          val_pos<PHASE>(n, g, c, t, row, p);
          val[q][n] = (use && t < R) ? __ldcg(sp + (t * NPROJ + p) * 32 + row) : 0.f;
        }
      }
#pragma unroll
      for (int q = 0; q < 4; ++q)
        if (q0 + q < W.on)
#pragma unroll
          for (int n = 0; n < NV; ++n) o.v[n] += val[q][n];
    }
  } else {
    // the contributors are the next non-empty warps of the grid, in atom order
    const int B1 = B0 + l.NA;
    int w = W.gw + 1;             // next candidate warp
    int at = W.part.atom_at(w);   // its first atom
    while (at < B1) {
      // up to four contributors' slots in flight, added in order
      int sid[4];
      int nq = 0;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        sid[q] = -1;
        if (at < B1) {
          int nx = W.part.atom_at(w + 1);
          while (nx == at) {  // warps with empty ranges hold nothing
            ++w;
            nx = W.part.atom_at(w + 1);
          }
          sid[q] = w;
          ++nq;
          ++w;
          at = nx;
        }
      }
      float val[4][NV];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float* sp = l.part + size_t(sid[q] < 0 ? 0 : sid[q]) * kSlotF;
#pragma unroll
        for (int n = 0; n < NV; ++n) {
          int t, row, p;
          val_pos<PHASE>(n, g, c, t, row, p);
          val[q][n] = (sid[q] >= 0 && t < R) ? __ldcg(sp + (t * NPROJ + p) * 32 + row) : 0.f;
        }
      }
#pragma unroll
      for (int q = 0; q < 4; ++q)
        if (q < nq)
#pragma unroll
          for (int n = 0; n < NV; ++n) o.v[n] += val[q][n];
    }
  }
  block_store<PHASE, NT>(a, m, v, t0, R, rb, lane, o);
  __syncwarp();
  if (lane == 0) *reinterpret_cast<volatile uint32_t*>(l.cnt + blk) = 0u;
  return true;
}

// Tensor maps of the code matrices: the routed experts' projections, then
// the shared expert's (phase 0: gate, up, shared gate, shared up; phase 1:
// down, shared down).
struct LaneMaps {
  CUtensorMap m[4];
  CUtensorMap s[4];  // the matching scale matrices (boxes of 32 rows x 16 bytes)
};

template <int PHASE>
__global__ void __launch_bounds__(LaneCfg<PHASE == 0 ? 2 : 1>::THREADS, 1)
    k_ffn_mma(const __grid_constant__ FfnArgs a, const __grid_constant__ LaneArgs l,
              const __grid_constant__ LaneMaps maps) {
  constexpr int NPROJ = PHASE == 0 ? 2 : 1;
  using C = LaneCfg<NPROJ>;
  constexpr int kLW = C::NW;
  constexpr int kLThreads = C::THREADS;
  extern __shared__ __align__(16) unsigned char lane_smem[];
  const uint32_t raw = lsm(lane_smem);
  unsigned char* codes = lane_smem + (((raw + C::HEAD + 1023u) & ~1023u) - raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(lane_smem);
  int* s_pfx = reinterpret_cast<int*>(lane_smem + C::SLOTS * 8);  // [kPfxMax]
  int* s_cpfx = s_pfx + kPfxMax;                                  // [kPfxMax]
  int* s_rv = s_cpfx + kPfxMax;                                   // [kPfxMax]
  int* s_plan = s_rv + kPfxMax;                                   // [kPfxMax]
  int* s_off = s_plan + kPfxMax;                                  // [kPfxMax]
  int* s_wsum = s_off + kPfxMax;                                  // [kLW][2]
  int* s_ent = s_wsum + 2 * kLW;                                  // [kEntMax]
  int* s_own = s_ent + kEntMax;                                   // [kLW][kOwnMax]
  uint8_t* s_xe = reinterpret_cast<uint8_t*>(s_own + kLW * kOwnMax);  // [kLaneMaxT]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tid = threadIdx.x;

  LaneWarp<PHASE> W;
  W.a = &a;
  W.l = &l;
  W.maps = maps.m;
  W.smaps = maps.s;
  W.codes = codes + size_t(warp) * C::WARP_BYTES;
  W.scales = W.codes + C::D * C::SLOT;
  W.exps = W.scales + C::NSCE * C::SCE;
  W.ri = C::NSCE - 1;
  W.sring = 0;
  W.full = bars + warp * C::D;
  if (lane == 0) {
    // arrivals: the expect_tx arrive, plus one per lane with cp.async scales
    const uint32_t count = l.sbox ? 1u : 33u;
    for (int d = 0; d < C::D; ++d)
      asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(lsm(&W.full[d])), "r"(count));
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  // The down projection's routing data (plan, buckets) and weights are ready
  // before the previous kernel (gate/up) ends: its setup and first weight
  // loads run ahead of the wait; only its operand rows (h) wait.
  if constexpr (PHASE == 0) pdl_wait();
  pdl_trigger();

  // Routing metadata and the workspace's wait limit and debug switches: one
  // round of independent loads into shared memory / registers.
  const int npairs = a.T * a.k;
  const bool ent_smem = npairs <= kEntMax;
  const unsigned wait_us = __ldg(reinterpret_cast<const unsigned*>(a.err) + 2);
  const unsigned debug = __ldg(reinterpret_cast<const unsigned*>(a.err) + 3);
  for (int i = tid; i < a.E + 2; i += kLThreads) s_plan[i] = __ldg(a.plan + i);
  for (int i = tid; i <= a.E; i += kLThreads) s_off[i] = __ldg(a.offsets + i);
  if (ent_smem)
    for (int i = tid; i < npairs; i += kLThreads) s_ent[i] = __ldg(a.entries + i);
  if constexpr (PHASE == 0)
    for (int i = tid; i < a.T; i += kLThreads) s_xe[i] = __ldg(a.xexp + i);
  __syncthreads();
  Meta meta;
  meta.plan = s_plan;
  meta.off = s_off;
  meta.ent = ent_smem ? s_ent : a.entries;
  meta.rv = s_rv;
  meta.xe = s_xe;
  meta.nA = s_plan[0];
  meta.nV = meta.nA + (a.has_shared ? 1 : 0);
  meta.T = a.T;
  meta.k = a.k;
  W.m = &meta;

  W.K = PHASE == 0 ? a.H : a.I;
  W.ROWS = PHASE == 0 ? a.I : a.H;
  W.nb = W.K / 32;
  W.nV = meta.nV;
  W.lane = lane;
  W.jc = W.ji = 0;
  W.pend = W.ppar = 0;
  W.iv = -1;
  W.ipass = -1;
  W.irows = 0;
  W.ixsrc = nullptr;
  W.iesrc = nullptr;
  W.iseg = -1;
  W.islot = W.cslot = 0;
  W.cpar = 0;
  W.wait_ns = (wait_us ? wait_us : kDefaultWaitUs) * 1000ull;

  // Per virtual expert: tokens, passes and cost; prefix sums over the
  // experts (two entries per thread).
  {
    int np[2] = {0, 0}, cu[2] = {0, 0};
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int v = 2 * tid + i;
      if (v < W.nV) {
        int R = a.T;
        if (v < meta.nA) {
          const int e = s_plan[1 + v];
          R = s_off[e + 1] - s_off[e];
        }
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
  W.pfx = s_pfx;
  const int NWtot = gridDim.x * kLW;
  W.part.init(s_pfx, s_cpfx, s_rv, W.nV, l.RB * l.NA, NWtot);

  W.gw = blockIdx.x * kLW + warp;
  const int A0 = W.part.atom_at(W.gw), A1 = W.part.atom_at(W.gw + 1);
  W.starve = (debug & MOE_DEBUG_STARVE_FIRST_WAIT) != 0 && PHASE == 0 && W.gw == 0;
  if (A0 >= A1) {
    if constexpr (PHASE == 1) pdl_wait();
    return;
  }

  LaneIt cur;
  it_begin(cur, A0, A1, l, W.pfx, W.nV);
  it_begin(W.nxt, A0, A1, l, W.pfx, W.nV);
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

  // While the first stages are in flight: list the contributors of the split
  // row block this warp will own at the end of its range.
  W.on = -1;
  W.osid = s_own + warp * kOwnMax;
  {
    const int NA = l.NA;
    const int lb0 = (A1 - 1) / NA * NA;  // first atom of the last row block
    if (lb0 >= A0 && A1 - lb0 < NA) {
      // lanes look up the next warps' first atoms in parallel; the
      // contributors are the non-empty ones among them, in order
      const int B1 = lb0 + NA;
      int n = 0, w = W.gw + 1;
      int at = A1;  // first atom of warp w
      bool done = false;
      while (!done && n < kOwnMax) {
        const int nx = W.part.atom_at(w + 1 + lane);  // first atom of warp w + 1 + lane
        const int cur_at = __shfl_up_sync(kFull, nx, 1);
        const int my_at = lane == 0 ? at : cur_at;    // first atom of warp w + lane
        const bool member = my_at < B1 && nx > my_at;  // non-empty and inside the block
        const unsigned mm = __ballot_sync(kFull, member);
        const int slot = n + __popc(mm & ((1u << lane) - 1u));
        if (member && slot < kOwnMax) W.osid[slot] = w + lane;
        n += __popc(mm);
        const unsigned past = __ballot_sync(kFull, nx >= B1);
        done = past != 0;
        at = __shfl_sync(kFull, nx, 31);
        w += 32;
      }
      __syncwarp();
      if (done && n <= kOwnMax) W.on = n;
    }
  }

  const FragOfs f = frag_ofs(lane);
  bool ok = true;
  while (ok && cur.valid) {
    if constexpr (PHASE == 0) {
      ok = run_pass<0, 1>(W, cur, f);
    } else {
      // two column tiles (hi/lo of 8 tokens) only for passes of more than 4
      if (meta.rv[cur.v] - cur.pass * kRMax <= 4) ok = run_pass<1, 1>(W, cur, f);
      else ok = run_pass<1, 2>(W, cur, f);
    }
  }
  if (!ok) W.drain();
}

template <int PHASE>
cudaError_t launch_mma_phase(const FfnArgs& a, const LaneArgs& l, const LaneMaps& maps,
                             cudaStream_t st) {
  using C = LaneCfg<PHASE == 0 ? 2 : 1>;
  auto kern = k_ffn_mma<PHASE>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  const int grid = device_info().sm_count < kLaneMaxCtas ? device_info().sm_count : kLaneMaxCtas;
  return launch_pdl(kern, dim3(grid), dim3(C::THREADS), size_t(C::SMEM), st, a, l, maps);
}

}  // namespace

bool lane_supported(const moe_shape_t& s) {
  // whole 128-value atoms in both phases
  const int smem = LaneCfg<2>::SMEM > LaneCfg<1>::SMEM ? LaneCfg<2>::SMEM : LaneCfg<1>::SMEM;
  // the per-expert tables hold 256 routed experts and the shared one
  const bool prefix_fits = s.E + 2 <= kPfxMax;
  return s.T <= kLaneMaxT && s.H % kAtomVals == 0 && s.I % kAtomVals == 0 && prefix_fits &&
         device_info().max_smem_optin >= smem;
}

cudaError_t launch_ffn_lane(const FfnArgs& a, float* lane_part, uint32_t* lane_cnt,
                            cudaStream_t st) {
  moe_shape_t s{a.T, a.H, a.I, a.E, a.k};
  if (!lane_supported(s) || a.xh == nullptr || a.xexp == nullptr) return cudaErrorNotSupported;
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
  // scale bytes by TMA boxes where a row's scale bytes are a multiple of 16
  const uint64_t HS = uint64_t(a.H) / 32, IS = uint64_t(a.I) / 32;
  const int sbox0 = HS % 16 == 0, sbox1 = IS % 16 == 0;
  if (sbox0) {
    ok = make_tma_map_u8_plain(&g.s[0], a.ex.gs, HS, uint64_t(a.E) * a.I, 16, 32) &&
         make_tma_map_u8_plain(&g.s[1], a.ex.us, HS, uint64_t(a.E) * a.I, 16, 32);
    if (a.has_shared)
      ok = ok && make_tma_map_u8_plain(&g.s[2], a.sh.gs, HS, a.I, 16, 32) &&
           make_tma_map_u8_plain(&g.s[3], a.sh.us, HS, a.I, 16, 32);
    else {
      g.s[2] = g.s[0];
      g.s[3] = g.s[1];
    }
  }
  if (sbox1) {
    ok = ok && make_tma_map_u8_plain(&d.s[0], a.ex.ds, IS, uint64_t(a.E) * a.H, 16, 32);
    if (a.has_shared) ok = ok && make_tma_map_u8_plain(&d.s[1], a.sh.ds, IS, a.H, 16, 32);
    else d.s[1] = d.s[0];
  }
  if (!ok) return cudaErrorNotSupported;
  LaneArgs l0{lane_part, lane_cnt, a.H / kAtomVals, a.I / 32, sbox0};
  LaneArgs l1{lane_part, lane_cnt, a.I / kAtomVals, a.H / 32, sbox1};
  cudaError_t e = launch_mma_phase<0>(a, l0, g, st);
  if (e != cudaSuccess) return e;
  return launch_mma_phase<1>(a, l1, d, st);
}

}  // namespace moe
