// Slot bank: routed experts paged from pinned host memory into a bounded set
// of device expert slots, the experts of each call chosen by its router.
//
// The ds4-ssd engine keeps the routed experts outside device memory and
// streams the ones the router picks into a fixed slot bank ("ds4-ssd"
// README, "Run SSD Sidecar Mode": an expert cache of a set size, the routed
// MXFP4 experts read on demand; "Experimental Pro Support": the shared
// expert's down projection prefetched).  Here the backing store is pinned
// host memory and the bank a caller-owned device region of n_slots experts;
// the shared expert stays resident (the caller passes it as usual).
//
// A banked call: router + top-k on the device; the chosen expert ids come
// back to the host (the one synchronisation of the call); the host makes them
// resident -- slots of experts already there are reused, missing experts
// take the least recently used slots not needed by this call, one
// cudaMemcpyAsync per matrix -- and writes the expert -> slot map; a kernel
// rewrites the indices to slot ids; bucket, expert FFNs and combine then run
// unchanged over the bank (E = n_slots).  The combine weights follow the
// (token, slot) pairs, so the output is the layer's.
#include <cstring>
#include <new>
#include <vector>

#include "moe_internal.cuh"

namespace moe {
namespace {

__global__ void __launch_bounds__(256) k_remap(const int32_t* idx, const int32_t* map, int n,
                                               int E, int32_t* out, int* err) {
  pdl_wait();
  pdl_trigger();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const int e = idx[i];
  const int s = (e >= 0 && e < E) ? map[e] : -1;
  if (s < 0) latch_error(err, MOE_ERR_DEVICE_DATA, 600 + (i & 63));
  out[i] = s;
}

}  // namespace
}  // namespace moe

using namespace moe;

struct moe_slot_bank {
  moe_mxfp4_experts_t host;  // E experts, pinned host memory
  int32_t H, I, E, n_slots;
  unsigned char* mem;        // device: n_slots experts in the canonical layout
  size_t mat_q, mat_s;       // bytes of one projection's codes / scales
  std::vector<int32_t> slot_owner;  // expert in each slot, -1 free
  std::vector<int32_t> expert_slot; // slot of each expert, -1 not resident
  std::vector<int64_t> last_use;    // call counter of the slot's last use
  int64_t clock;
  int64_t hits, misses, evictions;
  int32_t* map_host;         // pinned: expert -> slot for the map copy
  int32_t* ids_host;         // pinned: the call's expert ids
};

namespace {

size_t expert_bytes_of(int32_t H, int32_t I) {
  return 3 * (size_t(H) * I / 2 + size_t(H) * I / 32);
}

// The six projection arrays of slot s inside the bank's memory.
void slot_ptrs(const moe_slot_bank* b, int s, unsigned char* p[6]) {
  const size_t n = size_t(b->n_slots);
  unsigned char* base = b->mem;
  const size_t q = b->mat_q, sc = b->mat_s;
  p[0] = base + s * q;                                   // gate_q [n, I, H/2]
  p[1] = base + n * q + s * sc;                          // gate_s
  p[2] = base + n * (q + sc) + s * q;                    // up_q
  p[3] = base + n * (2 * q + sc) + s * sc;               // up_s
  p[4] = base + n * (2 * q + 2 * sc) + s * q;            // down_q [n, H, I/2]
  p[5] = base + n * (3 * q + 2 * sc) + s * sc;           // down_s
}

}  // namespace

extern "C" {

size_t moe_slot_bank_bytes(int32_t H, int32_t I, int32_t n_slots) {
  if (H < 32 || I < 32 || H % 32 || I % 32 || n_slots < 1) return 0;
  return size_t(n_slots) * expert_bytes_of(H, I);
}

moe_status_t moe_slot_bank_create(const moe_mxfp4_experts_t* host_experts, int32_t H, int32_t I,
                                  int32_t n_slots, void* slot_mem, size_t slot_mem_bytes,
                                  moe_slot_bank_t** out) {
  if (out == nullptr || host_experts == nullptr) return MOE_ERR_INVALID_ARG;
  *out = nullptr;
  const size_t need = moe_slot_bank_bytes(H, I, n_slots);
  if (need == 0 || host_experts->n_experts < 1 || host_experts->n_experts > kMaxExperts)
    return MOE_ERR_UNSUPPORTED_SHAPE;
  if (slot_mem == nullptr || (reinterpret_cast<uintptr_t>(slot_mem) & 15u)) return MOE_ERR_INVALID_ARG;
  if (slot_mem_bytes < need) return MOE_ERR_WORKSPACE;
  const void* hp[6] = {host_experts->gate_q, host_experts->gate_s, host_experts->up_q,
                       host_experts->up_s, host_experts->down_q, host_experts->down_s};
  for (const void* p : hp)
    if (p == nullptr) return MOE_ERR_INVALID_ARG;
  moe_slot_bank* b = new (std::nothrow) moe_slot_bank();
  if (b == nullptr) return MOE_ERR_WORKSPACE;
  b->host = *host_experts;
  b->H = H;
  b->I = I;
  b->E = host_experts->n_experts;
  b->n_slots = n_slots;
  b->mem = static_cast<unsigned char*>(slot_mem);
  b->mat_q = size_t(H) * I / 2;
  b->mat_s = size_t(H) * I / 32;
  b->slot_owner.assign(n_slots, -1);
  b->expert_slot.assign(b->E, -1);
  b->last_use.assign(n_slots, -1);
  b->clock = 0;
  b->hits = b->misses = b->evictions = 0;
  if (cudaMallocHost(&b->map_host, size_t(b->E) * 4) != cudaSuccess ||
      cudaMallocHost(&b->ids_host, size_t(kLaneMaxT) * kMaxTopK * 4) != cudaSuccess) {
    cudaGetLastError();
    delete b;
    return MOE_ERR_CUDA;
  }
  *out = b;
  return MOE_OK;
}

void moe_slot_bank_destroy(moe_slot_bank_t* b) {
  if (b == nullptr) return;
  cudaFreeHost(b->map_host);
  cudaFreeHost(b->ids_host);
  delete b;
}

moe_status_t moe_slot_bank_experts(const moe_slot_bank_t* b, moe_mxfp4_experts_t* out) {
  if (b == nullptr || out == nullptr) return MOE_ERR_INVALID_ARG;
  unsigned char* p[6];
  slot_ptrs(b, 0, p);
  out->gate_q = p[0];
  out->gate_s = p[1];
  out->up_q = p[2];
  out->up_s = p[3];
  out->down_q = p[4];
  out->down_s = p[5];
  out->n_experts = b->n_slots;
  return MOE_OK;
}

moe_status_t moe_slot_bank_acquire(moe_slot_bank_t* b, const int32_t* ids, int32_t n,
                                   int32_t* slot_of, void* stream) {
  if (b == nullptr || (n > 0 && (ids == nullptr || slot_of == nullptr)) || n < 0)
    return MOE_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t now = ++b->clock;
  // distinct experts of the call, and the resident ones marked as in use
  std::vector<int32_t> need;
  int distinct = 0;
  std::vector<char> seen(b->E, 0);
  for (int i = 0; i < n; ++i) {
    const int e = ids[i];
    if (e < 0 || e >= b->E) return MOE_ERR_INVALID_ARG;
    if (seen[e]) continue;
    seen[e] = 1;
    ++distinct;
    const int sl = b->expert_slot[e];
    if (sl >= 0) {
      b->last_use[sl] = now;
      ++b->hits;
    } else {
      need.push_back(e);
    }
  }
  if (distinct > b->n_slots) return MOE_ERR_WORKSPACE;
  // missing experts: the least recently used slots this call does not use
  for (int e : need) {
    int victim = -1;
    for (int sl = 0; sl < b->n_slots; ++sl) {
      if (b->last_use[sl] == now) continue;
      if (victim < 0 || b->last_use[sl] < b->last_use[victim]) victim = sl;
    }
    if (victim < 0) return MOE_ERR_WORKSPACE;  // cannot happen: distinct <= n_slots
    if (b->slot_owner[victim] >= 0) {
      b->expert_slot[b->slot_owner[victim]] = -1;
      ++b->evictions;
    }
    b->slot_owner[victim] = e;
    b->expert_slot[e] = victim;
    b->last_use[victim] = now;
    ++b->misses;
    unsigned char* dst[6];
    slot_ptrs(b, victim, dst);
    const unsigned char* src[6] = {
        b->host.gate_q + size_t(e) * b->mat_q, b->host.gate_s + size_t(e) * b->mat_s,
        b->host.up_q + size_t(e) * b->mat_q,   b->host.up_s + size_t(e) * b->mat_s,
        b->host.down_q + size_t(e) * b->mat_q, b->host.down_s + size_t(e) * b->mat_s};
    const size_t bytes[6] = {b->mat_q, b->mat_s, b->mat_q, b->mat_s, b->mat_q, b->mat_s};
    for (int m = 0; m < 6; ++m)
      if (cudaMemcpyAsync(dst[m], src[m], bytes[m], cudaMemcpyHostToDevice, s) != cudaSuccess) {
        cudaGetLastError();
        return MOE_ERR_CUDA;
      }
  }
  for (int i = 0; i < n; ++i) slot_of[i] = b->expert_slot[ids[i]];
  return MOE_OK;
}

moe_status_t moe_slot_bank_stats(const moe_slot_bank_t* b, int64_t* hits, int64_t* misses,
                                 int64_t* evictions) {
  if (b == nullptr) return MOE_ERR_INVALID_ARG;
  if (hits) *hits = b->hits;
  if (misses) *misses = b->misses;
  if (evictions) *evictions = b->evictions;
  return MOE_OK;
}

moe_status_t moe_layer_forward_banked(const uint16_t* x, const float* w_router, const float* bias,
                                      moe_slot_bank_t* bank, const moe_mxfp4_experts_t* shared,
                                      moe_shape_t shape, int32_t path, int32_t precision,
                                      uint16_t* y, int32_t* topk_idx_out, float* topk_w_out,
                                      void* ws, size_t ws_bytes, void* stream) {
  if (bank == nullptr) return MOE_ERR_INVALID_ARG;
  if (shape.E != bank->E || shape.H != bank->H || shape.I != bank->I) return MOE_ERR_INVALID_ARG;
  if (size_t(shape.T) * shape.k > size_t(kLaneMaxT) * kMaxTopK) return MOE_ERR_UNSUPPORTED_SHAPE;
  moe_shape_t sb = shape;
  sb.E = bank->n_slots;  // bucket, FFNs and combine run over the slots
  if (moe_workspace_bytes(shape, MOE_PATH_GEMV, MOE_ACT_EXACT, 0) == 0 ||
      moe_workspace_bytes(sb, path, precision, shared != nullptr) == 0)
    return MOE_ERR_UNSUPPORTED_SHAPE;
  const WsLayout Lr = ws_layout(shape, 0, 0);
  const WsLayout L = ws_layout(sb, shared != nullptr, path != MOE_PATH_GEMV);
  // the slot-id indices and the expert -> slot map sit after both layouts
  const size_t base = align256(Lr.total > L.total ? Lr.total : L.total);
  const size_t npairs = size_t(shape.T) * shape.k;
  const size_t map_at = base, sidx_at = align256(base + size_t(shape.E) * 4);
  const size_t need = align256(sidx_at + npairs * 4);
  if (ws == nullptr || ws_bytes < need) return MOE_ERR_WORKSPACE;
  if (topk_idx_out == nullptr || topk_w_out == nullptr) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  unsigned char* w8 = static_cast<unsigned char*>(ws);
  // 1. route (router + top-k) over all E experts
  moe_status_t st = moe_route_topk(x, w_router, bias, shape, nullptr, topk_idx_out, topk_w_out, ws,
                                   ws_bytes, stream);
  if (st != MOE_OK) return st;
  // 2. the chosen experts to the host; make them resident
  if (cudaMemcpyAsync(bank->ids_host, topk_idx_out, npairs * 4, cudaMemcpyDeviceToHost, s) !=
          cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  std::vector<int32_t> slots(npairs);
  st = moe_slot_bank_acquire(bank, bank->ids_host, int32_t(npairs), slots.data(), stream);
  if (st != MOE_OK) return st;
  for (int e = 0; e < bank->E; ++e) bank->map_host[e] = bank->expert_slot[e];
  int32_t* map_dev = reinterpret_cast<int32_t*>(w8 + map_at);
  int32_t* sidx = reinterpret_cast<int32_t*>(w8 + sidx_at);
  if (cudaMemcpyAsync(map_dev, bank->map_host, size_t(bank->E) * 4, cudaMemcpyHostToDevice, s) !=
      cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  // 3. expert ids -> slot ids
  cudaError_t e = launch_pdl(k_remap, dim3(unsigned((npairs + 255) / 256)), dim3(256), 0, s,
                             static_cast<const int32_t*>(topk_idx_out),
                             static_cast<const int32_t*>(map_dev), int(npairs), bank->E, sidx,
                             reinterpret_cast<int*>(w8 + L.err));
  if (e != cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  // 4. bucket, expert FFNs and combine over the slot bank
  int32_t* counts = reinterpret_cast<int32_t*>(w8 + L.counts);
  int32_t* offsets = reinterpret_cast<int32_t*>(w8 + L.offsets);
  int32_t* entries = reinterpret_cast<int32_t*>(w8 + L.entries);
  st = moe_bucket(sidx, sb, counts, offsets, entries, ws, ws_bytes, stream);
  if (st != MOE_OK) return st;
  moe_mxfp4_experts_t bank_ex;
  moe_slot_bank_experts(bank, &bank_ex);
  float* partial = reinterpret_cast<float*>(w8 + L.partial);
  st = moe_expert_ffn_mxfp4(&bank_ex, shared, x, offsets, entries, sb, path, precision, partial, ws,
                            ws_bytes, stream);
  if (st != MOE_OK) return st;
  return moe_combine(partial, topk_w_out, sb, shared != nullptr, y, stream);
}

size_t moe_layer_forward_banked_workspace_bytes(moe_shape_t shape, int32_t n_slots, int32_t path,
                                                int32_t precision, int32_t has_shared) {
  moe_shape_t sb = shape;
  sb.E = n_slots;
  const size_t a = moe_workspace_bytes(shape, MOE_PATH_GEMV, MOE_ACT_EXACT, 0);
  const size_t b = moe_workspace_bytes(sb, path, precision, has_shared);
  if (a == 0 || b == 0) return 0;
  const size_t base = align256(a > b ? a : b);
  return align256(align256(base + size_t(shape.E) * 4) + size_t(shape.T) * shape.k * 4);
}

}  // extern "C"
