// Grouped expert FFN on the 5th-generation tensor cores: block-scaled MXFP4
// x MXFP4 -> float32 (tcgen05.mma kind::mxf4, one E8M0 scale per 32 values
// on both operands), for prefill-sized batches.
//
// The pages run prefill chunks of up to 4K tokens ("ds4-ssd" README,
// "Validate": 4K prefill chunk cap) and route them through accelerator
// matmul paths on activations converted for the accelerator ("ds4-ssd"
// README, "Attribution": GPU dequantisation/packing feeding the ANE routed
// MLP; intro: NAX matmul2d).  Here the activations are quantised to MXFP4
// (OCP MX v1.0 rule) so both operands feed the FP4 tensor cores.
//
// Per virtual expert v (the activated routed experts in id order, then the
// shared expert) and per 128-row tile of its weights, one work item computes
//   D[m, n] = sum_k W[m, k] * A[n, k]      m: weight rows, n: bucket tokens
// with W on the MMA's M side (128 rows) and the bucket's tokens on its N side
// (up to BN per item), so small buckets waste no tensor work on padding.
// Two TMEM accumulator buffers let the epilogue of one item overlap the MMAs
// of the next.
// Phase 0: W = gate and up (two accumulators), epilogue h = silu(g) * u,
// re-quantised to MXFP4 along I.  Phase 1: W = down, epilogue writes the
// float32 expert outputs into `partial` rows (pair index order).
//
// CTA roles (224 threads, one persistent CTA per SM):
//   warp 0      TMA producer: weight and activation tiles (128-byte swizzle,
//               no multicast), one arrival with the transaction bytes per
//               stage;
//   warp 6      scale producer: the E8M0 scale bytes of each pair of stages
//               (16 bytes of every row), loaded into registers one pair ahead
//               and written as whole rows of the tcgen05 scale-factor atom
//               layout (byte 16*(r%32) + 4*(r/32%4) + k of a 512-byte atom
//               holds the scale of row r, K-block k); the next work item's
//               weight-scale block is prefetched into L2;
//   warp 1      TMEM allocation; lane 0 issues tcgen05.cp (scales -> TMEM)
//               and tcgen05.mma, and commits stage / accumulator barriers;
//   warps 2..5  epilogue: tcgen05.ld of their 32-lane TMEM quarter.
// Each stage's full barrier completes on the tile bytes plus the scale
// warp's arrival; both producers wait on its empty barrier.
// Every mbarrier wait is bounded (globaltimer); on expiry the CTA latches
// MOE_ERR_TIMEOUT in the workspace, drains what it issued and exits.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int kBM = 128;            // weight rows per item (MMA M)
constexpr int kBKB = 128;           // K bytes per stage (256 FP4 values)
constexpr int kGemmThreads = 224;
constexpr unsigned long long kWaitNs = 2000000000ull;  // default bound of a wait: 2 s
constexpr int kSmallN = 16;         // token rows of the small activation box

template <int PHASE>
struct GemmCfg {
  static constexpr int NPROJ = PHASE == 0 ? 2 : 1;
  // bucket tokens per item (MMA N); two accumulator buffers of NPROJ x BN
  // columns plus the scale factors fit the 512 TMEM columns
  static constexpr int BN = PHASE == 0 ? 112 : 128;
  static constexpr int NMB = (BN + 127) / 128;   // 128-row blocks of B scale factors
  static constexpr int A_BYTES = kBM * kBKB;     // 16 KB per projection
  static constexpr int B_BYTES = BN * kBKB;
  static constexpr int SFA_BYTES = 2 * 512;      // two K atoms (8 scales) per stage
  static constexpr int SFB_BYTES = 2 * NMB * 512;
  static constexpr int STAGE_RAW = NPROJ * A_BYTES + B_BYTES + NPROJ * SFA_BYTES + SFB_BYTES;
  static constexpr int STAGE = (STAGE_RAW + 1023) / 1024 * 1024;
  static constexpr int EPI_BYTES = PHASE == 0 ? 4 * 32 * 33 * 4 : 0;  // transpose tiles
  static constexpr int BUDGET = 216 * 1024 - EPI_BYTES;
  static constexpr int NS = BUDGET / STAGE > 8 ? 8 : BUDGET / STAGE;
  static constexpr int SMEM = NS * STAGE + EPI_BYTES + 1024 /*barriers*/ + 1024 /*alignment*/;
  // plus, after SMEM, the per-virtual-expert routing tables (tables_bytes)
  // TMEM columns: two accumulator buffers, then scale factors
  static constexpr int ACC_COLS = NPROJ * BN;
  static constexpr int SFA_COL = 2 * ACC_COLS;              // NPROJ * 8 columns
  static constexpr int SFB_COL = SFA_COL + NPROJ * 8;       // 2 * NMB * 4 columns
  static constexpr int USED_COLS = SFB_COL + 2 * NMB * 4;
  static constexpr int TMEM_COLS = USED_COLS <= 32 ? 32 : USED_COLS <= 64 ? 64
                                 : USED_COLS <= 128 ? 128 : USED_COLS <= 256 ? 256 : 512;
  static_assert(USED_COLS <= 512, "TMEM budget");
  static_assert(NS >= 2, "pipeline depth");
};

struct GemmArgs {
  const int32_t* offsets;
  const int32_t* entries;
  const int32_t* plan;
  const int32_t* item_off;  // [nV + 1] items before virtual expert v
  const uint8_t* sa[2];     // weight scales of the routed experts [E*ROWS, K/32]
  const uint8_t* sa_sh[2];  // weight scales of the shared expert [ROWS, K/32]
  const uint8_t* sb;        // activation scales [rows, K/32]
  uint8_t* hq;              // phase 0 output codes  [rows, I/2]
  uint8_t* hs;              // phase 0 output scales [rows, I/32]
  float* partial;           // phase 1 output [T*k + S*T, H]
  int* err;
  int T, H, I, E, k, has_shared;
};

// ------------------------------------------------------------ primitives ---
__device__ __forceinline__ uint32_t saddr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ unsigned long long globaltimer() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
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
// Bounded wait (limit_ns); false if it gave up (or another role already
// did).  Called by one lane; warp_wait() makes the outcome uniform over a warp.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort,
                                          int* err, int where, unsigned long long limit_ns) {
  if (mbar_try(bar, parity)) return true;
  const unsigned long long t0 = globaltimer();
  while (!mbar_try(bar, parity)) {
    if (*abort) return false;
    if (globaltimer() - t0 > limit_ns) {
      *abort = 1;
      latch_error(err, MOE_ERR_TIMEOUT, where);
      return false;
    }
  }
  return true;
}
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* abort,
                                          int* err, int where, unsigned long long limit_ns) {
  int ok = 0;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, abort, err, where, limit_ns);
  return __shfl_sync(kFull, ok, 0) != 0;
}
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}
// The same with an L2 cache policy (expert weights: read once per call,
// evict first, so they do not push the activations, the router weights and
// the workspace out of L2).
__device__ __forceinline__ void tma_load_2d_hint(uint32_t dst, const CUtensorMap* map, int x, int y,
                                                 uint32_t bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar), "l"(policy)
      : "memory");
}
__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
// word q (0..3) of a uint4
__device__ __forceinline__ uint32_t u4_word(const uint4& v, int q) {
  return q == 0 ? v.x : q == 1 ? v.y : q == 2 ? v.z : v.w;
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}
// 32 rows x 16 bytes of scale factors (one 512-byte atom) -> 4 TMEM columns,
// replicated into the four 32-lane quarters.
__device__ __forceinline__ void tc_cp_sf(uint32_t tmem, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(tmem), "l"(sdesc)
               : "memory");
}
__device__ __forceinline__ void tc_mma_mxf4(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc,
                                            uint32_t accumulate, uint32_t sfa, uint32_t sfb) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
      ::"r"(d), "l"(a), "l"(b), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
      : "memory");
}

// Shared-memory matrix descriptor: K-major operand, 128-byte swizzle, rows of
// 128 bytes, 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t desc_sw128(uint32_t addr) {
  return uint64_t((addr & 0x3FFFFu) >> 4) | (uint64_t(1) << 16) | (uint64_t(1024 >> 4) << 32) |
         (uint64_t(1) << 46) | (uint64_t(2) << 61);
}
// Descriptor of one scale-factor atom: 32 rows of 16 bytes, no swizzle.
__device__ __forceinline__ uint64_t desc_sf(uint32_t addr) {
  return uint64_t((addr & 0x3FFFFu) >> 4) | (uint64_t(128 >> 4) << 32) | (uint64_t(1) << 46);
}
// Instruction descriptor: kind::mxf4, E2M1 x E2M1, E8M0 scales, K-major A/B,
// M = 128, N = n, scale byte pair sf_id for both operands.
__device__ __forceinline__ uint32_t idesc_mxf4(int n, int sf_id) {
  return (1u << 7) | (1u << 10) | (uint32_t(n >> 3) << 17) | (1u << 23) | (uint32_t(kBM >> 4) << 24) |
         (uint32_t(sf_id) << 29) | (uint32_t(sf_id) << 4);
}

// 32 columns of this warp's TMEM quarter -> registers
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// ------------------------------------------------------------- work items ---
struct Item {
  int v;        // virtual expert
  int e;        // routed expert id, or -1 for the shared expert
  int mt, nt;   // weight row tile, token tile
  int row0;     // first activation row of the bucket
  int R;        // bucket tokens
  int nvalid;   // tokens of this item
};

// Per-virtual-expert routing tables, staged in shared memory once per CTA:
// items before v (nV + 1 entries), expert id (or -1), first activation row
// and tokens of v.
struct Tables {
  const int* item_off;
  const int* e;
  const int* row0;
  const int* R;
};
__host__ __device__ inline size_t tables_bytes(int E) { return size_t(4) * 4 * (E + 2); }

template <int BN>
__device__ __forceinline__ Item item_of(const Tables& tb, int it, int nV, int MT) {
  // virtual expert: last v with item_off[v] <= it
  int lo = 0, hi = nV - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (tb.item_off[mid] <= it) lo = mid;
    else hi = mid - 1;
  }
  Item r;
  r.v = lo;
  const int li = it - tb.item_off[lo];
  const int ntiles = (tb.item_off[lo + 1] - tb.item_off[lo]) / MT;
  r.mt = li / ntiles;
  r.nt = li % ntiles;  // token tiles fastest: neighbours share the weight tile in L2
  r.e = tb.e[lo];
  r.row0 = tb.row0[lo];
  r.R = tb.R[lo];
  r.nvalid = min(BN, r.R - r.nt * BN);
  return r;
}

// ------------------------------------------------------------------ kernel ---
template <int PHASE>
__global__ void __launch_bounds__(kGemmThreads, 1)
    k_ffn_gemm(GemmArgs a, const __grid_constant__ CUtensorMap mA0,
               const __grid_constant__ CUtensorMap mA1, const __grid_constant__ CUtensorMap mS0,
               const __grid_constant__ CUtensorMap mS1, const __grid_constant__ CUtensorMap mB,
               const __grid_constant__ CUtensorMap mBs) {
  using C = GemmCfg<PHASE>;
  constexpr int NPROJ = C::NPROJ;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* epi = reinterpret_cast<float*>(smem + C::NS * C::STAGE);  // phase 0 transpose tiles
  unsigned char* ctl = smem + C::NS * C::STAGE + C::EPI_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(ctl);
  uint64_t* empty = full + C::NS;
  uint64_t* acc_full = empty + C::NS;   // [2]
  uint64_t* acc_empty = acc_full + 2;   // [2]
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* s_tab = reinterpret_cast<int*>(smem + C::SMEM - 1024);  // after the barriers' kilobyte

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(saddr(&full[s]), 2);  // TMA arrival + scales staged
      mbar_init(saddr(&empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(saddr(&acc_full[b]), 1);
      mbar_init(saddr(&acc_empty[b]), 4);
    }
    mbar_init(saddr(drain), 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     saddr(tmem_slot)),
                 "r"(C::TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (threadIdx.x == 0) {
    // the descriptors are fetched while the previous kernel drains
    const void* maps[6] = {&mA0, &mA1, &mS0, &mS1, &mB, &mBs};
#pragma unroll
    for (int i = 0; i < 6; ++i) asm volatile("prefetch.tensormap [%0];" ::"l"(maps[i]) : "memory");
  }

  pdl_wait();
  pdl_trigger();
  // the workspace's wait limit (0: the default) and debug switches
  const unsigned wait_us = __ldg(reinterpret_cast<const unsigned*>(a.err) + 2);
  const unsigned debug = __ldg(reinterpret_cast<const unsigned*>(a.err) + 3);
  const unsigned long long wait_ns = wait_us ? wait_us * 1000ull : kWaitNs;

  // routing tables -> shared memory (one round of loads)
  Tables tb;
  {
    const int nA0 = __ldg(a.plan);
    const int nV0 = nA0 + (a.has_shared ? 1 : 0);
    int* t_off = s_tab;
    int* t_e = t_off + (a.E + 2);
    int* t_row0 = t_e + (a.E + 2);
    int* t_R = t_row0 + (a.E + 2);
    for (int v = threadIdx.x; v <= nV0; v += blockDim.x) {
      t_off[v] = __ldg(a.item_off + v);
      if (v < nA0) {
        const int e = __ldg(a.plan + 1 + v);
        const int r0 = __ldg(a.offsets + e);
        t_e[v] = e;
        t_row0[v] = r0;
        t_R[v] = __ldg(a.offsets + e + 1) - r0;
      } else if (v < nV0) {
        t_e[v] = -1;
        t_row0[v] = a.T * a.k;
        t_R[v] = a.T;
      }
    }
    __syncthreads();
    tb.item_off = t_off;
    tb.e = t_e;
    tb.row0 = t_row0;
    tb.R = t_R;
  }

  const int K = PHASE == 0 ? a.H : a.I;
  const int ROWS = PHASE == 0 ? a.I : a.H;
  const int KB = K / 2;        // bytes per row
  const int NSC = K / 32;      // scale bytes per row
  const int nks = (KB + kBKB - 1) / kBKB;
  const int MT = ROWS / kBM;
  const int nA = __ldg(a.plan);
  const int nV = nA + (a.has_shared ? 1 : 0);
  const int n_items = tb.item_off[nV];

  const int my_items = n_items > int(blockIdx.x) ? (n_items - 1 - int(blockIdx.x)) / int(gridDim.x) + 1 : 0;
  const int total = my_items * nks;  // stages of this CTA, numbered g = 0..

  if (warp == 0) {
    // ------------------------------------------------------- tile producer
    // Items of at most kSmallN tokens load a kSmallN-row activation box
    // instead of BN rows.
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t fills = 0;  // bit s: parity of the last fill of stage s
      uint32_t used = 0;   // bit s: stage s was filled at least once
      uint64_t pol;
      asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
      Item w{};
      int arow = 0, brow = 0;
      for (int g = 0; g < total; ++g) {
        const int ks = g % nks;
        if (ks == 0) {
          w = item_of<C::BN>(tb, int(blockIdx.x) + (g / nks) * int(gridDim.x), nV, MT);
          arow = (w.e >= 0 ? w.e * ROWS : 0) + w.mt * kBM;
          brow = w.row0 + w.nt * C::BN;
        }
        const bool routed = w.e >= 0;
        const bool small = w.nvalid <= kSmallN;
        if (!mbar_wait(saddr(&empty[stage]), phase ^ 1u, abort_flag, a.err, 100, wait_ns)) break;
        unsigned char* st = smem + stage * C::STAGE;
        const uint32_t fb = saddr(&full[stage]);
        if (PHASE == 0 && g == 0 && blockIdx.x == 0 && (debug & MOE_DEBUG_STARVE_FIRST_WAIT)) {
          // debug switch: the first stage gets no tile copies, so the MMA
          // thread's bounded wait on it runs out
          if (++stage == C::NS) {
            stage = 0;
            phase ^= 1u;
          }
          continue;
        }
        mbar_expect_tx(fb, NPROJ * C::A_BYTES + (small ? kSmallN : C::BN) * kBKB);
        tma_load_2d_hint(saddr(st), routed ? &mA0 : &mS0, ks * kBKB, arow, fb, pol);
        if constexpr (NPROJ == 2)
          tma_load_2d_hint(saddr(st + C::A_BYTES), routed ? &mA1 : &mS1, ks * kBKB, arow, fb, pol);
        tma_load_2d(saddr(st + NPROJ * C::A_BYTES), small ? &mBs : &mB, ks * kBKB, brow, fb);
        fills ^= 1u << stage;  // parity of this fill's phase = bit after toggle ^ 1
        used |= 1u << stage;
        if (++stage == C::NS) {
          stage = 0;
          phase ^= 1u;
        }
      }
      // after a give-up, let every tile this thread requested land (bounded)
      if (*abort_flag) {
        for (int s = 0; s < C::NS; ++s) {
          if (!((used >> s) & 1u)) continue;
          const uint32_t last_parity = ((fills >> s) & 1u) ^ 1u;
          const unsigned long long t0 = globaltimer();
          while (!mbar_try(saddr(&full[s]), last_parity) && globaltimer() - t0 < 100000000ull) {
          }
        }
      }
    }
    __syncwarp();
  } else if (warp == 6) {
    // ------------------------------------------------------ scale producer
    // The stages of an item are taken in pairs (the last one alone when nks
    // is odd).  Lane l holds rows l, l+32, l+64, l+96 of each operand; word q
    // of a row's 16 bytes is stage q/2 of the pair, atom q%2.
    constexpr int NBJ = C::NMB * 4;  // 32-row groups of B scale rows
    int stage = 0;
    uint32_t phase = 0;
    const bool vec16 = (NSC & 15) == 0;  // rows start 16-byte aligned
    // the weight-scale block of item li of this CTA (128 contiguous rows of
    // NSC bytes per projection) -> L2, an item ahead of its first use
    auto prefetch_item = [&](int li) {
      if (lane != 0 || li >= my_items) return;
      const Item x = item_of<C::BN>(tb, int(blockIdx.x) + li * int(gridDim.x), nV, MT);
      const size_t off = (size_t(x.e >= 0 ? x.e * ROWS : 0) + size_t(x.mt) * kBM) * NSC;
#pragma unroll
      for (int p = 0; p < NPROJ; ++p)
        asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"((x.e >= 0 ? a.sa[p] : a.sa_sh[p]) + off),
                     "r"(uint32_t(kBM * NSC))
                     : "memory");
    };
    Item wn{};
    int arow_n = 0, brow_n = 0;
    uint4 sa_n[NPROJ][4], sb_n[NBJ];
    auto load_pair = [&](int g_n) {
      const int ks_n = g_n % nks;
      if (ks_n == 0) {
        wn = item_of<C::BN>(tb, int(blockIdx.x) + (g_n / nks) * int(gridDim.x), nV, MT);
        arow_n = (wn.e >= 0 ? wn.e * ROWS : 0) + wn.mt * kBM;
        brow_n = wn.row0 + wn.nt * C::BN;
        prefetch_item(g_n / nks + 1);
      }
      const int c0 = ks_n * 8;  // first scale byte of the pair
      // words past the end of a row (the tail of K) read as zero scales:
      // their K blocks are never multiplied
      auto row16 = [&](const uint8_t* rowp) {
        if (vec16 && c0 + 16 <= NSC) return __ldg(reinterpret_cast<const uint4*>(rowp + c0));
        uint32_t v[4];
#pragma unroll
        for (int q = 0; q < 4; ++q)
          v[q] = c0 + 4 * q + 4 <= NSC ? __ldg(reinterpret_cast<const uint32_t*>(rowp + c0 + 4 * q)) : 0u;
        return make_uint4(v[0], v[1], v[2], v[3]);
      };
#pragma unroll
      for (int p = 0; p < NPROJ; ++p) {
        const uint8_t* src = wn.e >= 0 ? a.sa[p] : a.sa_sh[p];
#pragma unroll
        for (int j = 0; j < 4; ++j) sa_n[p][j] = row16(src + size_t(arow_n + lane + 32 * j) * NSC);
      }
#pragma unroll
      for (int j = 0; j < NBJ; ++j) {
        const int n = lane + 32 * j;
        sb_n[j] = n < wn.nvalid ? row16(a.sb + size_t(brow_n + n) * NSC) : make_uint4(0, 0, 0, 0);
      }
    };
    prefetch_item(0);
    if (total > 0) load_pair(0);
    for (int g = 0; g < total;) {
      const int ks = g % nks;
      const int npair = ks + 1 < nks ? 2 : 1;
      uint4 sa[NPROJ][4], sb[NBJ];
#pragma unroll
      for (int p = 0; p < NPROJ; ++p)
#pragma unroll
        for (int j = 0; j < 4; ++j) sa[p][j] = sa_n[p][j];
#pragma unroll
      for (int j = 0; j < NBJ; ++j) sb[j] = sb_n[j];
      if (g + npair < total) load_pair(g + npair);
      const int slot0 = stage;
      const uint32_t phase0 = phase;
      if (++stage == C::NS) {
        stage = 0;
        phase ^= 1u;
      }
      const int slot1 = stage;
      const uint32_t phase1 = phase;
      if (npair == 2 && ++stage == C::NS) {
        stage = 0;
        phase ^= 1u;
      }
      if (!warp_wait(saddr(&empty[slot0]), phase0 ^ 1u, abort_flag, a.err, 110, wait_ns)) break;
      if (npair == 2 && !warp_wait(saddr(&empty[slot1]), phase1 ^ 1u, abort_flag, a.err, 111, wait_ns)) break;
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        if (u == npair) break;
        unsigned char* sfa = smem + (u ? slot1 : slot0) * C::STAGE + NPROJ * C::A_BYTES + C::B_BYTES;
        unsigned char* sfb = sfa + NPROJ * C::SFA_BYTES;
#pragma unroll
        for (int at = 0; at < 2; ++at) {
          const int q = 2 * u + at;
#pragma unroll
          for (int p = 0; p < NPROJ; ++p)
            *reinterpret_cast<uint4*>(sfa + p * C::SFA_BYTES + at * 512 + 16 * lane) =
                make_uint4(u4_word(sa[p][0], q), u4_word(sa[p][1], q), u4_word(sa[p][2], q),
                           u4_word(sa[p][3], q));
#pragma unroll
          for (int mb = 0; mb < C::NMB; ++mb)
            *reinterpret_cast<uint4*>(sfb + at * C::NMB * 512 + mb * 512 + 16 * lane) =
                make_uint4(u4_word(sb[4 * mb], q), u4_word(sb[4 * mb + 1], q),
                           u4_word(sb[4 * mb + 2], q), u4_word(sb[4 * mb + 3], q));
        }
      }
      fence_proxy_async();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(saddr(&full[slot0]));
        if (npair == 2) mbar_arrive(saddr(&full[slot1]));
      }
      g += npair;
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------------- MMA
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      const uint32_t tsfa = tmem + C::SFA_COL;
      const uint32_t tsfb = tmem + C::SFB_COL;
      int local = 0;  // items of this CTA so far: buffer local & 1, use local >> 1
      for (int it = blockIdx.x; it < n_items && ok; it += gridDim.x, ++local) {
        const Item w = item_of<C::BN>(tb, it, nV, MT);
        const int n_mma = ((w.nvalid + 7) / 8) * 8;
        const int buf = local & 1;
        const uint32_t acc_parity = (uint32_t(local >> 1) & 1u) ^ 1u;
        if (!mbar_wait(saddr(&acc_empty[buf]), acc_parity, abort_flag, a.err, 200, wait_ns)) break;
        tc_fence_after();
        const uint32_t tacc = tmem + buf * C::ACC_COLS;
        for (int ks = 0; ks < nks; ++ks) {
          if (!mbar_wait(saddr(&full[stage]), phase, abort_flag, a.err, 201, wait_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          unsigned char* st = smem + stage * C::STAGE;
          unsigned char* sfa = st + NPROJ * C::A_BYTES + C::B_BYTES;
          unsigned char* sfb = sfa + NPROJ * C::SFA_BYTES;
#pragma unroll
          for (int p = 0; p < NPROJ; ++p)
#pragma unroll
            for (int at = 0; at < 2; ++at)
              tc_cp_sf(tsfa + p * 8 + at * 4, desc_sf(saddr(sfa + p * C::SFA_BYTES + at * 512)));
#pragma unroll
          for (int at = 0; at < 2; ++at)
#pragma unroll
            for (int mb = 0; mb < C::NMB; ++mb)
              tc_cp_sf(tsfb + (at * C::NMB + mb) * 4,
                       desc_sf(saddr(sfb + at * C::NMB * 512 + mb * 512)));
          const int kb_n = min(4, (KB - ks * kBKB) / 32);  // 64-value K blocks in this stage
          for (int kb = 0; kb < kb_n; ++kb) {
            const uint32_t id = idesc_mxf4(n_mma, (kb & 1) * 2);
            const uint64_t bdesc = desc_sw128(saddr(st + NPROJ * C::A_BYTES) + kb * 32);
#pragma unroll
            for (int p = 0; p < NPROJ; ++p) {
              const uint64_t adesc = desc_sw128(saddr(st + p * C::A_BYTES) + kb * 32);
              tc_mma_mxf4(tacc + p * C::BN, adesc, bdesc, id, (ks | kb) != 0,
                          tsfa + p * 8 + (kb >> 1) * 4, tsfb + (kb >> 1) * C::NMB * 4);
            }
          }
          tc_commit(saddr(&empty[stage]));
          if (++stage == C::NS) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit(saddr(&acc_full[buf]));
      }
      if (!ok || *abort_flag) {
        // give-up path: let issued MMAs finish before TMEM is released
        tc_commit(saddr(drain));
        const unsigned long long t0 = globaltimer();
        while (!mbar_try(saddr(drain), 0) && globaltimer() - t0 < 200000000ull) {
        }
      }
    }
    __syncwarp();
  } else if (warp >= 2 && warp <= 5) {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    float* tile = epi + q * 32 * 33;  // 32 x 32 transpose tile (phase 0)
    int local = 0;
    for (int it = blockIdx.x; it < n_items; it += gridDim.x, ++local) {
      const Item w = item_of<C::BN>(tb, it, nV, MT);
      const int buf = local & 1;
      if (!warp_wait(saddr(&acc_full[buf]), uint32_t(local >> 1) & 1u, abort_flag, a.err, 300, wait_ns))
        break;
      tc_fence_after();
      const uint32_t tacc = tmem + buf * C::ACC_COLS;
      const int wrow = w.mt * kBM + 32 * q + lane;  // weight row of this lane
      for (int c0 = 0; c0 < w.nvalid; c0 += 32) {
        const uint32_t taddr = tacc + (uint32_t(32 * q) << 16) + c0;
        if constexpr (PHASE == 0) {
          // h for 32 tokens of this lane's row, transposed through shared
          // memory so each thread holds one token's 32 consecutive h values:
          // exactly one MXFP4 block along I, quantised in registers
          float g[32], u[32];
          tmem_ld32(taddr, g);
          tmem_ld32(taddr + C::BN, u);
#pragma unroll
          for (int j = 0; j < 32; ++j) tile[lane * 33 + j] = g[j] / (1.f + expf(-g[j])) * u[j];
          __syncwarp();
          const int n = c0 + lane;  // token of this thread
          if (n < w.nvalid) {
            float hv[32];
            float amax = 0.f;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              hv[i] = tile[i * 33 + lane];
              amax = fmaxf(amax, fabsf(hv[i]));
            }
            const int X = mx_scale_exponent(amax);
            const float inv = exp2i(-X);
            uint32_t word[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              uint32_t acc = 0;
#pragma unroll
              for (int b = 0; b < 4; ++b)
                acc |= f32x2_to_e2m1x2(hv[8 * j + 2 * b] * inv, hv[8 * j + 2 * b + 1] * inv)
                       << (8 * b);
              word[j] = acc;
            }
            const size_t orow = size_t(w.row0 + w.nt * C::BN + n);
            const int i0 = w.mt * kBM + 32 * q;  // first intermediate index of the block
            *reinterpret_cast<uint4*>(a.hq + orow * (a.I / 2) + i0 / 2) =
                make_uint4(word[0], word[1], word[2], word[3]);
            a.hs[orow * (a.I / 32) + i0 / 32] = uint8_t(X + 127);
          }
          __syncwarp();
        } else {
          // partial rows of the chunk's 32 tokens: one coalesced load, then
          // broadcast, so the stores do not wait on index loads one by one
          const int nl = c0 + lane;
          int prow_l = 0;
          if (nl < w.nvalid) {
            const int r = w.nt * C::BN + nl;
            prow_l = w.e >= 0 ? __ldg(a.entries + w.row0 + r) : a.T * a.k + r;
          }
          float o[32];
          tmem_ld32(taddr, o);
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int prow = __shfl_sync(kFull, prow_l, j);
            if (c0 + j < w.nvalid) a.partial[size_t(prow) * a.H + wrow] = o[j];
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(saddr(&acc_empty[buf]));
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(C::TMEM_COLS)
                 : "memory");
  }
}

// ---------------------------------------------------- activation gather ---
// Row r < T*k of the gathered operand is token entries[r] / k (bucket order);
// rows T*k + t are token t (shared expert).  One warp per row.
__global__ void __launch_bounds__(256) k_act_gather(const uint16_t* x, const int32_t* entries,
                                                    int T, int H, int k, int rows, uint8_t* q,
                                                    uint8_t* s) {
  pdl_wait();
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = blockIdx.x * 8 + warp;
  if (r >= rows) return;
  const int tok = r < T * k ? entries[r] / k : r - T * k;
  const uint16_t* src = x + size_t(tok) * H;
  const int nb = H / 32;
  for (int b = lane; b < nb; b += 32) {
    const uint4* p = reinterpret_cast<const uint4*>(src + size_t(b) * 32);
    float f[32];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint4 v = __ldg(p + j);
      const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        f[8 * j + 2 * i] = bf16_bits_to_f32(wv[i] & 0xffffu);
        f[8 * j + 2 * i + 1] = bf16_bits_to_f32(wv[i] >> 16);
      }
    }
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(f[i]));
    const int X = mx_scale_exponent(amax);
    const float inv = exp2i(-X);
    uint32_t word[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint32_t acc = 0;
#pragma unroll
      for (int i = 0; i < 4; ++i)
        acc |= f32x2_to_e2m1x2(f[8 * j + 2 * i] * inv, f[8 * j + 2 * i + 1] * inv) << (8 * i);
      word[j] = acc;
    }
    *reinterpret_cast<uint4*>(q + size_t(r) * (H / 2) + size_t(b) * 16) =
        make_uint4(word[0], word[1], word[2], word[3]);
    s[size_t(r) * nb + b] = uint8_t(X + 127);
  }
}

// ------------------------------------------------------- item prefix sums ---
// item_off[p][v] = sum_{v' < v} MT_p * ceil(R_v' / BN_p) for both phases.
__global__ void __launch_bounds__(1024) k_gemm_plan(const int32_t* offsets, const int32_t* plan,
                                                    int T, int k, int has_shared, int MT0, int MT1,
                                                    int32_t* item_off0, int32_t* item_off1) {
  pdl_wait();
  pdl_trigger();
  constexpr int BN0 = GemmCfg<0>::BN, BN1 = GemmCfg<1>::BN;
  __shared__ int rows_of[kMaxExperts + 2];
  const int nA = plan[0];
  const int nV = nA + (has_shared ? 1 : 0);
  for (int v = threadIdx.x; v < nV; v += blockDim.x) {
    if (v < nA) {
      const int e = plan[1 + v];
      rows_of[v] = offsets[e + 1] - offsets[e];
    } else {
      rows_of[v] = T;
    }
  }
  __syncthreads();
  if (threadIdx.x < 32) {
    // one warp: running prefix sums in chunks of 32
    int run0 = 0, run1 = 0;
    for (int base = 0; base < nV; base += 32) {
      const int v = base + threadIdx.x;
      const int R = v < nV ? rows_of[v] : 0;
      const int t0 = (R + BN0 - 1) / BN0 * MT0, t1 = (R + BN1 - 1) / BN1 * MT1;
      int i0 = t0, i1 = t1;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int y0 = __shfl_up_sync(kFull, i0, off), y1 = __shfl_up_sync(kFull, i1, off);
        if ((int)threadIdx.x >= off) {
          i0 += y0;
          i1 += y1;
        }
      }
      if (v < nV) {
        item_off0[v] = run0 + i0 - t0;
        item_off1[v] = run1 + i1 - t1;
      }
      run0 += __shfl_sync(kFull, i0, 31);
      run1 += __shfl_sync(kFull, i1, 31);
    }
    if (threadIdx.x == 0) {
      item_off0[nV] = run0;
      item_off1[nV] = run1;
    }
  }
}

// --------------------------------------------------------------- host side ---
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    cudaDriverEntryPointQueryResult q{};
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 2-D map of a [rows, row_bytes] uint8 matrix, boxes of box_rows x 128 bytes.
bool make_map(CUtensorMap* m, const void* base, uint64_t row_bytes, uint64_t rows,
              uint32_t box_rows) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {row_bytes, rows};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {uint32_t(kBKB), box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int PHASE>
cudaError_t launch_gemm_phase(const GemmArgs& g, const CUtensorMap& a0, const CUtensorMap& a1,
                              const CUtensorMap& s0, const CUtensorMap& s1, const CUtensorMap& b,
                              const CUtensorMap& bs, cudaStream_t st) {
  using C = GemmCfg<PHASE>;
  auto kern = k_ffn_gemm<PHASE>;
  const size_t smem = size_t(C::SMEM) + tables_bytes(g.E);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, dim3(device_info().sm_count), dim3(kGemmThreads), smem, st, g, a0, a1, s0,
                    s1, b, bs);
}

}  // namespace

// 2-D map of a [rows, row_bytes] uint8 matrix, boxes of box_rows x box_bytes
// (64 or 128) with the swizzle of the same width (the decode GEMV's
// code boxes).
bool make_tma_map_u8_box(CUtensorMap* m, const void* base, uint64_t row_bytes, uint64_t rows,
                         uint32_t box_bytes, uint32_t box_rows) {
  auto fn = encode_fn();
  if (fn == nullptr || (box_bytes != 64 && box_bytes != 128)) return false;
  const cuuint64_t dims[2] = {row_bytes, rows};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_bytes, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE,
            box_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D map of a [rows, row_bytes] uint8 matrix (row_bytes a multiple of 16),
// boxes of box_rows x box_bytes, no swizzle (the decode GEMV's scale boxes).
bool make_tma_map_u8_plain(CUtensorMap* m, const void* base, uint64_t row_bytes, uint64_t rows,
                           uint32_t box_bytes, uint32_t box_rows) {
  auto fn = encode_fn();
  if (fn == nullptr || row_bytes % 16 != 0 || box_bytes % 16 != 0) return false;
  const cuuint64_t dims[2] = {row_bytes, rows};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_bytes, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool gemm_supported(const moe_shape_t& s) {
  // the routing tables of E experts share the opt-in shared memory (227 KB)
  // with the pipeline stages
  const size_t cap = 227 * 1024, tab = tables_bytes(s.E);
  return s.H % 256 == 0 && s.I % 128 == 0 && size_t(GemmCfg<0>::SMEM) + tab <= cap &&
         size_t(GemmCfg<1>::SMEM) + tab <= cap && encode_fn() != nullptr;
}

cudaError_t launch_ffn_gemm(const FfnArgs& a, const GemmBuffers& gb, cudaStream_t st) {
  const int rows = a.T * a.k + (a.has_shared ? a.T : 0);
  cudaError_t e = launch_pdl(k_act_gather, dim3((rows + 7) / 8), dim3(256), 0, st, a.x, a.entries,
                             a.T, a.H, a.k, rows, gb.xq, gb.xs);
  if (e != cudaSuccess) return e;
  e = launch_pdl(k_gemm_plan, dim3(1), dim3(1024), 0, st, a.offsets, a.plan, a.T, a.k,
                 a.has_shared, a.I / kBM, a.H / kBM, gb.item_off0, gb.item_off1);
  if (e != cudaSuccess) return e;

  CUtensorMap g0, g1, sg0, sg1, bx, bxs, d0, sd0, bh, bhs;
  const uint64_t HB = a.H / 2, IB = a.I / 2;
  bool ok = make_map(&g0, a.ex.gq, HB, uint64_t(a.E) * a.I, kBM) &&
            make_map(&g1, a.ex.uq, HB, uint64_t(a.E) * a.I, kBM) &&
            make_map(&bx, gb.xq, HB, rows, GemmCfg<0>::BN) &&
            make_map(&bxs, gb.xq, HB, rows, kSmallN) &&
            make_map(&d0, a.ex.dq, IB, uint64_t(a.E) * a.H, kBM) &&
            make_map(&bh, gb.hq, IB, rows, GemmCfg<1>::BN) &&
            make_map(&bhs, gb.hq, IB, rows, kSmallN);
  if (a.has_shared) {
    ok = ok && make_map(&sg0, a.sh.gq, HB, a.I, kBM) && make_map(&sg1, a.sh.uq, HB, a.I, kBM) &&
         make_map(&sd0, a.sh.dq, IB, a.H, kBM);
  } else {
    sg0 = g0;
    sg1 = g1;
    sd0 = d0;
  }
  if (!ok) return cudaErrorInvalidValue;

  GemmArgs g{};
  g.offsets = a.offsets;
  g.entries = a.entries;
  g.plan = a.plan;
  g.err = a.err;
  g.T = a.T;
  g.H = a.H;
  g.I = a.I;
  g.E = a.E;
  g.k = a.k;
  g.has_shared = a.has_shared;
  // phase 0: gate/up, SwiGLU, MXFP4 h
  g.item_off = gb.item_off0;
  g.sa[0] = a.ex.gs;
  g.sa[1] = a.ex.us;
  g.sa_sh[0] = a.has_shared ? a.sh.gs : a.ex.gs;
  g.sa_sh[1] = a.has_shared ? a.sh.us : a.ex.us;
  g.sb = gb.xs;
  g.hq = gb.hq;
  g.hs = gb.hs;
  e = launch_gemm_phase<0>(g, g0, g1, sg0, sg1, bx, bxs, st);
  if (e != cudaSuccess) return e;
  // phase 1: down
  g.item_off = gb.item_off1;
  g.sa[0] = a.ex.ds;
  g.sa[1] = a.ex.ds;
  g.sa_sh[0] = a.has_shared ? a.sh.ds : a.ex.ds;
  g.sa_sh[1] = g.sa_sh[0];
  g.sb = gb.hs;
  g.partial = a.partial;
  return launch_gemm_phase<1>(g, d0, d0, sd0, sd0, bh, bhs, st);
}

}  // namespace moe
