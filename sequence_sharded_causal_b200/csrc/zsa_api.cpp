// zsa_api.cpp -- the C ABI declared in include/zsa.h.
//
// Argument validation happens here, before anything is enqueued; every entry point
// returns a status code and nothing throws across the ABI.  The library allocates no
// device memory: the forward's unit table travels in the caller's workspace, copied
// from a pinned host copy that is cached per shape.
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstring>
#include <map>
#include <memory>
#include <mutex>
#include <set>
#include <tuple>
#include <utility>

#include "../../include/zsa.h"
#include "zsa_kernels.h"
#include "zsa_schedule.h"

namespace {

using zsa::Schedule;

constexpr size_t kStatusBytes = 256;
std::atomic<uint64_t> g_wait_limit_ns{2000000000ull};
std::atomic<int> g_inject_stall{0};
constexpr int kTraceKernels = 7;
std::atomic<void*> g_trace_begin[kTraceKernels];
std::atomic<void*> g_trace_end[kTraceKernels];

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

int check_problem(const zsa_problem* p) {
  if (!p) return ZSA_ERR_INVALID;
  if (p->B <= 0 || p->S <= 0 || p->Hq <= 0 || p->Hkv <= 0 || p->d <= 0 || p->D <= 0)
    return ZSA_ERR_INVALID;
  if (!(p->softmax_scale > 0.0f) || !std::isfinite(p->softmax_scale)) return ZSA_ERR_INVALID;
  if (p->causal != 0 && p->causal != 1) return ZSA_ERR_INVALID;
  if (p->kv_layout != ZSA_KV_NATURAL && p->kv_layout != ZSA_KV_SHARD_MAJOR) return ZSA_ERR_INVALID;
  if (p->shard_begin < 0 || p->shard_count < 0 || p->shard_begin >= p->D ||
      p->shard_begin + (p->shard_count ? p->shard_count : p->D) > p->D)
    return ZSA_ERR_INVALID;
  if (p->shard_count == 0 && p->shard_begin != 0) return ZSA_ERR_INVALID;
  if (p->Hq % p->Hkv != 0) return ZSA_ERR_SHAPE;
  if (p->S % (2 * int64_t(p->D) * 64) != 0) return ZSA_ERR_SHAPE;
  if (p->B * p->S >= (int64_t(1) << 31)) return ZSA_ERR_SHAPE;  // TMA row coordinates are int32
  return ZSA_OK;
}

int check_device_problem(const zsa_problem* p) {
  int rc = check_problem(p);
  if (rc) return rc;
  if (p->d != 64 && p->d != 128 && p->d != 256) return ZSA_ERR_UNSUPPORTED;
  int32_t bq, bk, slots;
  zsa::fwd_tiling(p->d, &bq, &bk, &slots);
  if (p->S / bk >= 65536) return ZSA_ERR_SHAPE;  // key-tile counts are packed in 16 bits
  return ZSA_OK;
}

bool aligned16(const void* x) { return (reinterpret_cast<uintptr_t>(x) & 15) == 0; }

// Shards a call computes, and its Q-layout rows (shards * B * 2C).
int32_t local_shards(const zsa_problem* p) { return p->shard_count ? p->shard_count : p->D; }
int64_t local_rows(const zsa_problem* p) { return int64_t(local_shards(p)) * p->B * (p->S / p->D); }

int check_sm100() {
  static std::mutex mu;
  static std::map<int, int> arch_ok;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ZSA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(mu);
  auto it = arch_ok.find(dev);
  if (it != arch_ok.end()) return it->second;
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return ZSA_ERR_CUDA;
  int v = (major == 10 && minor == 0) ? ZSA_OK : ZSA_ERR_UNSUPPORTED;
  arch_ok[dev] = v;
  return v;
}

// ------------------------------------------------------------------ schedule cache
struct CachedSchedule {
  Schedule sched;
  zsa::DevUnit* pinned = nullptr;  // page-locked copy of sched.units (or nullptr)
  ~CachedSchedule() {
    if (pinned) cudaFreeHost(pinned);
  }
};

using SchedKey = std::tuple<int64_t, int32_t, int32_t, int32_t, int32_t, int32_t, int32_t, int32_t,
                           int32_t, int32_t, int32_t>;

std::shared_ptr<CachedSchedule> get_schedule(int64_t S, int32_t D, int32_t B, int32_t Hq,
                                             int32_t Hkv, int32_t causal, int32_t bq, int32_t bk,
                                             int32_t slots, int32_t shard_begin,
                                             int32_t shard_count, bool want_pinned) {
  static std::mutex mu;
  static std::map<SchedKey, std::shared_ptr<CachedSchedule>> cache;
  SchedKey key{S, D, B, Hq, Hkv, causal, bq, bk, slots, shard_begin, shard_count};
  {
    std::lock_guard<std::mutex> lock(mu);
    auto it = cache.find(key);
    if (it != cache.end() && (!want_pinned || it->second->pinned)) return it->second;
  }
  auto e = std::make_shared<CachedSchedule>();
  if (!zsa::build_schedule(S, D, B, Hq, Hkv, causal, bq, bk, slots, shard_begin, shard_count,
                           &e->sched))
    return nullptr;
  if (want_pinned) {
    const size_t bytes = e->sched.units.size() * sizeof(zsa::DevUnit);
    void* h = nullptr;
    if (cudaHostAlloc(&h, bytes ? bytes : 1, cudaHostAllocDefault) != cudaSuccess) return nullptr;
    std::memcpy(h, e->sched.units.data(), bytes);
    e->pinned = static_cast<zsa::DevUnit*>(h);
  }
  std::lock_guard<std::mutex> lock(mu);
  auto& slot = cache[key];
  if (!slot || (want_pinned && !slot->pinned)) slot = e;
  return slot;
}

size_t fwd_workspace(const zsa_problem* p) {
  int32_t bq, bk, slots;
  zsa::fwd_tiling(p->d, &bq, &bk, &slots);
  const int64_t T = (p->S / p->D) / bq;
  const int64_t G = p->Hq / p->Hkv;
  const int64_t runs = (T * G + slots - 1) / slots;
  const int64_t units = p->B * p->Hkv * local_shards(p) * runs;
  return kStatusBytes + align256(size_t(units) * sizeof(zsa::DevUnit));
}

size_t bwd_workspace(const zsa_problem* p) {
  const size_t stats = size_t(local_rows(p)) * p->Hq * sizeof(float);  // -Delta, -lse log2 e
  const size_t dqacc = size_t(local_rows(p)) * p->Hq * p->d * sizeof(float);
  return kStatusBytes + 2 * align256(stats) + align256(dqacc);
}

}  // namespace

namespace zsa {
int ensure_smem_attr(const void* func, int bytes) {
  static std::mutex mu;
  static std::set<std::pair<const void*, int>> done;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return int(e);
  std::lock_guard<std::mutex> lock(mu);
  if (done.count({func, dev})) return int(cudaSuccess);
  e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return int(e);
  done.insert({func, dev});
  return int(cudaSuccess);
}

uint64_t wait_limit_ns() { return g_wait_limit_ns.load(); }
int inject_stall() { return g_inject_stall.load(); }

TraceEvents trace_events(int which) {
  TraceEvents t{nullptr, nullptr};
  if (which >= 0 && which < kTraceKernels) {
    t.begin = static_cast<cudaEvent_t>(g_trace_begin[which].load());
    t.end = static_cast<cudaEvent_t>(g_trace_end[which].load());
  }
  return t;
}
}  // namespace zsa

extern "C" {

int zsa_trace_events(int which, void* begin_event, void* end_event) {
  if (which < 0 || which >= kTraceKernels) return ZSA_ERR_INVALID;
  g_trace_begin[which].store(begin_event);
  g_trace_end[which].store(end_event);
  return ZSA_OK;
}

const char* zsa_status_string(int status) {
  switch (status) {
    case ZSA_OK: return "ok";
    case ZSA_ERR_INVALID: return "invalid argument";
    case ZSA_ERR_SHAPE: return "unsupported shape (S % (2*D*64), Hq % Hkv or size limits)";
    case ZSA_ERR_UNSUPPORTED: return "unsupported head dim or device (needs sm_100)";
    case ZSA_ERR_WORKSPACE: return "workspace or schedule capacity too small";
    case ZSA_ERR_CUDA: return "CUDA runtime error";
    case ZSA_ERR_TIMEOUT: return "a bounded device-side wait timed out";
    default: return "unknown status";
  }
}

int zsa_debug_inject_stall(int enable) {
  g_inject_stall.store(enable ? 1 : 0);
  return ZSA_OK;
}

int zsa_set_wait_limit_ns(uint64_t limit_ns) {
  g_wait_limit_ns.store(limit_ns);
  return ZSA_OK;
}

int zsa_partition(const zsa_problem* problem, zsa_tiling* tiling, int32_t* perm_host,
                  int32_t* inv_perm_host, int64_t* shard_tiles_host, zsa_work* sched_host,
                  int64_t cap, int64_t* n_work_out) {
  int rc = check_problem(problem);
  if (rc) return rc;
  if (!tiling) return ZSA_ERR_INVALID;
  int32_t bq = tiling->block_q, bk = tiling->block_k, slots = tiling->slots;
  if (bq == 0 || bk == 0 || slots == 0) {
    int32_t dq, dk, ds;
    zsa::fwd_tiling(problem->d, &dq, &dk, &ds);
    if (bq == 0) bq = dq;
    if (bk == 0) bk = dk;
    if (slots == 0) slots = ds;
  }
  const int64_t S = problem->S;
  const int32_t D = problem->D;
  if (bq < 0 || bk < 0 || (slots != 1 && slots != 2)) return ZSA_ERR_INVALID;
  if ((S / D) % bq != 0 || S % bk != 0) return ZSA_ERR_SHAPE;
  if (S / bk >= 65536) return ZSA_ERR_SHAPE;
  tiling->block_q = bq;
  tiling->block_k = bk;
  tiling->slots = slots;
  const int64_t C = S / (2 * int64_t(D));
  if (perm_host || inv_perm_host) {
    for (int32_t r = 0; r < D; ++r)
      for (int64_t j = 0; j < 2 * C; ++j) {
        const int64_t pos = zsa::zigzag_pos(C, D, r, j);
        if (perm_host) perm_host[r * 2 * C + j] = int32_t(pos);
        if (inv_perm_host) inv_perm_host[pos] = int32_t(r * 2 * C + j);
      }
  }
  if (!shard_tiles_host && !sched_host && !n_work_out) return ZSA_OK;
  auto cs = get_schedule(S, D, int32_t(problem->B), problem->Hq, problem->Hkv, problem->causal, bq,
                         bk, slots, problem->shard_begin, local_shards(problem), false);
  if (!cs) return ZSA_ERR_SHAPE;
  const Schedule& sc = cs->sched;
  if (shard_tiles_host)
    for (int32_t r = 0; r < D; ++r) shard_tiles_host[r] = sc.shard_tiles[size_t(r)];
  const int64_t n = int64_t(sc.units.size());
  if (n_work_out) *n_work_out = n;
  if (sched_host) {
    if (cap < n) return ZSA_ERR_WORKSPACE;
    for (int64_t i = 0; i < n; ++i) {
      const zsa::DevUnit& u = sc.units[size_t(i)];
      zsa_work& w = sched_host[i];
      w.shard = u.r; w.b = u.b; w.kv_head = u.g;
      w.q_tile0 = u.tile0; w.q_head0 = u.head0; w.q_tile1 = u.tile1; w.q_head1 = u.head1;
      w.k_tile_end0 = u.kend & 0xFFFF;
      w.k_tile_end1 = (u.kend >> 16) & 0xFFFF;
    }
  }
  return ZSA_OK;
}

int zsa_workspace_bytes(const zsa_problem* problem, int pass, size_t* bytes_out) {
  int rc = check_device_problem(problem);
  if (rc) return rc;
  if (!bytes_out || (pass != 0 && pass != 1)) return ZSA_ERR_INVALID;
  *bytes_out = pass == 0 ? fwd_workspace(problem) : bwd_workspace(problem);
  return ZSA_OK;
}

namespace {
// The forward over all keys (block == nullptr) or over one block of keys.
int attn_fwd_impl(const zsa_problem* problem, const zsa_key_block* block, const void* q,
                  const void* k, const void* v, void* o, float* lse, void* workspace,
                  size_t ws_bytes, void* cuda_stream) {
  int rc = check_device_problem(problem);
  if (rc) return rc;
  if (!q || !k || !v || !o || !lse || !workspace) return ZSA_ERR_INVALID;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255))
    return ZSA_ERR_INVALID;
  if (ws_bytes < fwd_workspace(problem)) return ZSA_ERR_WORKSPACE;
  rc = check_sm100();
  if (rc) return rc;
  int32_t bq, bk, slots;
  zsa::fwd_tiling(problem->d, &bq, &bk, &slots);
  auto cs = get_schedule(problem->S, problem->D, int32_t(problem->B), problem->Hq, problem->Hkv,
                         problem->causal, bq, bk, slots, problem->shard_begin,
                         local_shards(problem), true);
  if (!cs) return ZSA_ERR_CUDA;
  cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const size_t table = cs->sched.units.size() * sizeof(zsa::DevUnit);
  if (cudaMemsetAsync(ws, 0, kStatusBytes, stream) != cudaSuccess) return ZSA_ERR_CUDA;
  if (table &&
      cudaMemcpyAsync(ws + kStatusBytes, cs->pinned, table, cudaMemcpyHostToDevice, stream) !=
          cudaSuccess)
    return ZSA_ERR_CUDA;
  zsa::FwdArgs a;
  a.q = q; a.k = k; a.v = v; a.o = o; a.lse = lse;
  a.units = reinterpret_cast<const zsa::DevUnit*>(ws + kStatusBytes);
  a.n_units = int32_t(cs->sched.units.size());
  a.S = problem->S; a.B = int32_t(problem->B); a.Hq = problem->Hq; a.Hkv = problem->Hkv;
  a.d = problem->d; a.D = problem->D; a.causal = problem->causal;
  a.scale = problem->softmax_scale;
  a.kv_layout = problem->kv_layout;
  a.shard_begin = problem->shard_begin;
  a.shard_count = local_shards(problem);
  a.status = reinterpret_cast<int*>(ws);
  a.wait_limit_ns = g_wait_limit_ns.load();
  a.inject_stall = g_inject_stall.load();
  if (block) {
    a.key_block = 1;
    a.key_lo = int32_t(block->key_lo);
    a.key_hi = int32_t(block->key_hi);
    a.kv_rows_per_batch = int32_t(block->rows_per_batch);
    a.kv_row_offset = int32_t(block->row_offset);
    a.kv_rows = int32_t(block->rows);
  }
  if (zsa::launch_fwd(a, stream) != int(cudaSuccess)) return ZSA_ERR_CUDA;
  return ZSA_OK;
}

bool key_block_ok(const zsa_problem* p, const zsa_key_block* kb) {
  const int64_t lim = int64_t(1) << 31;
  if (kb->key_lo < 0 || kb->key_hi < kb->key_lo || kb->key_hi > p->S) return false;
  if (kb->rows <= 0 || kb->rows >= lim || kb->row_offset < 0 || kb->row_offset >= lim ||
      kb->rows_per_batch < 0 || kb->rows_per_batch >= lim)
    return false;
  const int64_t len = kb->key_hi - kb->key_lo;
  if (p->B > 1 && kb->rows_per_batch < len) return false;
  return (p->B - 1) * kb->rows_per_batch + kb->row_offset + len <= kb->rows;
}
}  // namespace

int zsa_attn_fwd(const zsa_problem* problem, const void* q, const void* k, const void* v,
                 void* o, float* lse, void* workspace, size_t ws_bytes, void* cuda_stream) {
  return attn_fwd_impl(problem, nullptr, q, k, v, o, lse, workspace, ws_bytes, cuda_stream);
}

int zsa_attn_fwd_block(const zsa_problem* problem, const zsa_key_block* block, const void* q,
                       const void* k, const void* v, void* o, float* lse, void* workspace,
                       size_t ws_bytes, void* cuda_stream) {
  if (!problem || !block) return ZSA_ERR_INVALID;
  const int rc = check_problem(problem);
  if (rc) return rc;
  if (!key_block_ok(problem, block)) return ZSA_ERR_INVALID;
  return attn_fwd_impl(problem, block, q, k, v, o, lse, workspace, ws_bytes, cuda_stream);
}

int zsa_attn_bwd(const zsa_problem* problem, const void* q, const void* k, const void* v,
                 const void* o, const float* lse, const void* dout, void* dq, void* dk, void* dv,
                 void* workspace, size_t ws_bytes, void* cuda_stream) {
  int rc = check_device_problem(problem);
  if (rc) return rc;
  if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv || !workspace)
    return ZSA_ERR_INVALID;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) ||
      !aligned16(dout) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255))
    return ZSA_ERR_INVALID;
  if (ws_bytes < bwd_workspace(problem)) return ZSA_ERR_WORKSPACE;
  rc = check_sm100();
  if (rc) return rc;
  cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const size_t stats = size_t(local_rows(problem)) * problem->Hq * sizeof(float);
  if (cudaMemsetAsync(ws, 0, kStatusBytes, stream) != cudaSuccess) return ZSA_ERR_CUDA;
  zsa::BwdArgs a;
  a.q = q; a.k = k; a.v = v; a.o = o; a.lse = lse; a.dout = dout;
  a.dq = dq; a.dk = dk; a.dv = dv;
  a.delta = reinterpret_cast<float*>(ws + kStatusBytes);
  a.nlse2 = reinterpret_cast<float*>(ws + kStatusBytes + align256(stats));
  a.dq_acc = reinterpret_cast<float*>(ws + kStatusBytes + 2 * align256(stats));
  a.S = problem->S; a.B = int32_t(problem->B); a.Hq = problem->Hq; a.Hkv = problem->Hkv;
  a.d = problem->d; a.D = problem->D; a.causal = problem->causal;
  a.scale = problem->softmax_scale;
  a.kv_layout = problem->kv_layout;
  a.shard_begin = problem->shard_begin;
  a.shard_count = local_shards(problem);
  a.status = reinterpret_cast<int*>(ws);
  a.wait_limit_ns = g_wait_limit_ns.load();
  a.inject_stall = g_inject_stall.load();
  const int e = zsa::launch_bwd(a, stream);
  if (e == int(cudaErrorNotSupported)) return ZSA_ERR_UNSUPPORTED;
  if (e != int(cudaSuccess)) return ZSA_ERR_CUDA;
  return ZSA_OK;
}

int zsa_permute(const zsa_problem* problem, int32_t heads, int32_t to_shard_major,
                const void* src, void* dst, void* cuda_stream) {
  if (!problem) return ZSA_ERR_INVALID;
  int rc = check_problem(problem);
  if (rc) return rc;
  if (problem->d <= 0 || problem->d % 8 != 0 || heads <= 0) return ZSA_ERR_INVALID;
  if (to_shard_major != 0 && to_shard_major != 1) return ZSA_ERR_INVALID;
  if (!src || !dst || !aligned16(src) || !aligned16(dst)) return ZSA_ERR_INVALID;
  const int64_t C = problem->S / (2 * int64_t(problem->D));
  const int64_t row_bytes = int64_t(heads) * problem->d * 2;
  // the two tensors must not overlap (the copy is not ordered)
  const uintptr_t nat_bytes = uintptr_t(problem->B * problem->S * row_bytes);
  const uintptr_t smj_bytes = uintptr_t(local_rows(problem) * row_bytes);
  const uintptr_t s0 = reinterpret_cast<uintptr_t>(src), d0 = reinterpret_cast<uintptr_t>(dst);
  const uintptr_t s_bytes = to_shard_major ? nat_bytes : smj_bytes;
  const uintptr_t d_bytes = to_shard_major ? smj_bytes : nat_bytes;
  if (s0 < d0 + d_bytes && d0 < s0 + s_bytes) return ZSA_ERR_INVALID;
  if (2 * int64_t(local_shards(problem)) * problem->B > 65535) return ZSA_ERR_SHAPE;  // grid.y
  rc = check_sm100();
  if (rc) return rc;
  zsa::PermuteArgs a;
  a.src = src;
  a.dst = dst;
  a.chunk_words = C * row_bytes / 16;
  a.B = int32_t(problem->B);
  a.D = problem->D;
  a.shard_begin = problem->shard_begin;
  a.shard_count = local_shards(problem);
  a.to_shard_major = to_shard_major;
  if (zsa::launch_permute(a, static_cast<cudaStream_t>(cuda_stream)) != int(cudaSuccess))
    return ZSA_ERR_CUDA;
  return ZSA_OK;
}

int zsa_attn_merge(const zsa_problem* problem, int32_t n_parts, const void* const* o_parts,
                   const float* const* lse_parts, void* o, float* lse, void* cuda_stream) {
  int rc = check_device_problem(problem);
  if (rc) return rc;
  if (n_parts < 1 || n_parts > ZSA_MERGE_MAX_PARTS || !o_parts || !lse_parts || !o || !lse)
    return ZSA_ERR_INVALID;
  if (local_rows(problem) * problem->Hq * problem->d >= (int64_t(1) << 31)) return ZSA_ERR_SHAPE;
  zsa::MergeArgs a;
  for (int i = 0; i < n_parts; ++i) {
    if (!o_parts[i] || !lse_parts[i] || !aligned16(o_parts[i]) || !aligned16(lse_parts[i]))
      return ZSA_ERR_INVALID;
    a.o[i] = o_parts[i];
    a.lse[i] = lse_parts[i];
  }
  if (!aligned16(o) || !aligned16(lse)) return ZSA_ERR_INVALID;
  rc = check_sm100();
  if (rc) return rc;
  a.o_out = o;
  a.lse_out = lse;
  a.S = problem->S;
  a.rows = local_rows(problem);
  a.Hq = problem->Hq; a.d = problem->d; a.D = problem->D; a.n = n_parts;
  if (zsa::launch_merge(a, static_cast<cudaStream_t>(cuda_stream)) != int(cudaSuccess))
    return ZSA_ERR_CUDA;
  return ZSA_OK;
}

int zsa_tsp_project(int64_t T, int64_t K, int64_t N, const void* x, int64_t ldx, const void* w,
                    int64_t ldw, const zsa_proj_segment* segs, int32_t n_segs, void* status_ws,
                    void* cuda_stream) {
  if (!x || !w || !segs || !status_ws) return ZSA_ERR_INVALID;
  if (T <= 0 || K <= 0 || N <= 0 || ldx < K || ldw < N) return ZSA_ERR_INVALID;
  if (N % 32 || K % 8) return ZSA_ERR_SHAPE;
  if (ldx % 8 || ldw % 8 || !aligned16(x) || !aligned16(w) ||
      (reinterpret_cast<uintptr_t>(status_ws) & 255))
    return ZSA_ERR_INVALID;
  if (T >= (int64_t(1) << 31) || K >= (int64_t(1) << 31) || N >= (int64_t(1) << 31))
    return ZSA_ERR_SHAPE;
  if (n_segs < 1 || n_segs > ZSA_PROJ_MAX_SEGMENTS) return ZSA_ERR_INVALID;
  zsa::ProjArgs a;
  int64_t col = 0;
  for (int i = 0; i < n_segs; ++i) {
    const zsa_proj_segment& g = segs[i];
    if (!g.out || g.cols <= 0 || g.cols % 32 || g.ld % 8 || !aligned16(g.out) ||
        (g.fp32_accumulate != 0 && g.fp32_accumulate != 1) || g.ld < g.cols)
      return ZSA_ERR_INVALID;
    a.segs[i].out = g.out;
    a.segs[i].ld = g.ld;
    a.segs[i].col_begin = col;
    a.segs[i].col_end = col + g.cols;
    a.segs[i].fp32_accumulate = g.fp32_accumulate;
    col += g.cols;
  }
  if (col != N) return ZSA_ERR_INVALID;
  int rc = check_sm100();
  if (rc) return rc;
  cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
  if (cudaMemsetAsync(status_ws, 0, kStatusBytes, stream) != cudaSuccess) return ZSA_ERR_CUDA;
  a.x = x; a.w = w;
  a.T = T; a.N = N; a.K = K; a.ldx = ldx; a.ldw = ldw;
  a.n_segs = n_segs;
  a.status = static_cast<int*>(status_ws);
  a.wait_limit_ns = g_wait_limit_ns.load();
  if (zsa::launch_proj_gemm(a, stream) != int(cudaSuccess)) return ZSA_ERR_CUDA;
  return ZSA_OK;
}

int zsa_device_status(void* workspace, void* cuda_stream) {
  if (!workspace) return ZSA_ERR_INVALID;
  cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
  int st = 0;
  if (cudaMemcpyAsync(&st, workspace, sizeof(int), cudaMemcpyDeviceToHost, stream) != cudaSuccess)
    return ZSA_ERR_CUDA;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return ZSA_ERR_CUDA;
  if (st == 0) return ZSA_OK;
  if (cudaMemsetAsync(workspace, 0, sizeof(int), stream) != cudaSuccess) return ZSA_ERR_CUDA;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return ZSA_ERR_CUDA;
  return ZSA_ERR_TIMEOUT;
}

}  // extern "C"
