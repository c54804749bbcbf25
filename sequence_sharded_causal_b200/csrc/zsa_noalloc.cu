// zsa_noalloc.cu -- the backward pass for callers that cannot allocate device memory.
//
// zsa_attn_bwd needs a caller-provided workspace (status word, -Delta, -lse*log2(e), fp32
// dQ accumulator).  Some callers have no way to provide one at the call site: plugins
// inside a host runtime whose device memory is entirely owned and pre-planned by that
// runtime (they may not call cudaMalloc, and the runtime offers no scratch hook), or a
// C caller that links the library without any allocator of its own.
// zsa_attn_bwd_noalloc serves them: its scratch is a file-scope __device__ array of
// fixed size (ZSA_NOALLOC_SCRATCH_BYTES), so the call itself allocates nothing.  The
// same backward kernels run; only the scratch pointers differ.
//
// Costs and rules, stated for users:
//  * every GPU on which this library's module is loaded keeps the array resident until
//    the process exits (with CUDA's eager module loading that is every GPU the process
//    creates a context on, whether or not it ever calls this entry point);
//  * problems whose scratch need (the same number zsa_workspace_bytes(problem, 1)
//    reports) exceeds ZSA_NOALLOC_SCRATCH_BYTES are rejected with ZSA_ERR_WORKSPACE
//    before anything is enqueued;
//  * all calls share the one array per device and it keeps the previous call's
//    contents: the dQ accumulator is zeroed by the preprocess kernel and the status
//    word by this entry point, on every call.  Calls whose GPU work overlaps (two
//    streams, or two host threads) race on the array and give wrong results;
//  * the first call on each device looks up the array's device address
//    (cudaGetSymbolAddress) with that device current; make that first call before
//    any stream capture begins;
//  * the wait limit and the stall hook (zsa_set_wait_limit_ns, zsa_debug_inject_stall)
//    apply as they do to zsa_attn_bwd; a wait that gives up records a timeout in the
//    status word inside the array, which zsa_noalloc_status reads and clears.
#include <cuda_runtime.h>

#include <cmath>
#include <cstring>
#include <mutex>

#include "../../include/zsa.h"
#include "zsa_kernels.h"

namespace {

constexpr size_t kNoAllocStatusBytes = 256;

// The scratch.  In host code this name is only a host-side stand-in for the symbol,
// never a device address: host code must use the address cudaGetSymbolAddress returns.
static __device__ __align__(256) unsigned char g_noalloc_scratch[ZSA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch on the current device (looked up once per device).
int scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ZSA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return ZSA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
      return ZSA_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return ZSA_OK;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

bool aligned16(const void* x) { return (reinterpret_cast<uintptr_t>(x) & 15) == 0; }

}  // namespace

extern "C" int zsa_attn_bwd_noalloc(const zsa_problem* problem, const void* q, const void* k,
                                    const void* v, const void* o, const float* lse,
                                    const void* dout, void* dq, void* dk, void* dv,
                                    void* cuda_stream) {
  // Shape, pointer and size checks happen before any CUDA call.
  size_t need = 0;
  int rc = zsa_workspace_bytes(problem, 1, &need);
  if (rc != ZSA_OK) return rc;
  if (need > size_t(ZSA_NOALLOC_SCRATCH_BYTES)) return ZSA_ERR_WORKSPACE;
  if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv) return ZSA_ERR_INVALID;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) ||
      !aligned16(dout) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return ZSA_ERR_INVALID;
  int major = 0, minor = 0, dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return ZSA_ERR_CUDA;
  if (major != 10 || minor != 0) return ZSA_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  rc = scratch_address(&scratch);
  if (rc != ZSA_OK) return rc;

  cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
  uint8_t* base = static_cast<uint8_t*>(scratch);
  if (cudaMemsetAsync(base, 0, kNoAllocStatusBytes, stream) != cudaSuccess) return ZSA_ERR_CUDA;
  const int32_t shards = problem->shard_count ? problem->shard_count : problem->D;
  const size_t stats =
      size_t(shards) * problem->B * (problem->S / problem->D) * problem->Hq * sizeof(float);
  zsa::BwdArgs a;
  a.q = q; a.k = k; a.v = v; a.o = o; a.lse = lse; a.dout = dout;
  a.dq = dq; a.dk = dk; a.dv = dv;
  a.delta = reinterpret_cast<float*>(base + kNoAllocStatusBytes);
  a.nlse2 = reinterpret_cast<float*>(base + kNoAllocStatusBytes + align256(stats));
  a.dq_acc = reinterpret_cast<float*>(base + kNoAllocStatusBytes + 2 * align256(stats));
  a.S = problem->S; a.B = int32_t(problem->B); a.Hq = problem->Hq; a.Hkv = problem->Hkv;
  a.d = problem->d; a.D = problem->D; a.causal = problem->causal;
  a.scale = problem->softmax_scale;
  a.kv_layout = problem->kv_layout;
  a.shard_begin = problem->shard_begin;
  a.shard_count = shards;
  a.status = reinterpret_cast<int*>(base);
  a.wait_limit_ns = zsa::wait_limit_ns();
  a.inject_stall = zsa::inject_stall();
  const int e = zsa::launch_bwd(a, stream);
  if (e == int(cudaErrorNotSupported)) return ZSA_ERR_UNSUPPORTED;
  if (e != int(cudaSuccess)) return ZSA_ERR_CUDA;
  return ZSA_OK;
}

extern "C" int zsa_noalloc_status(void* cuda_stream) {
  void* scratch = nullptr;
  int rc = scratch_address(&scratch);
  if (rc != ZSA_OK) return rc;
  cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
  int st = 0;
  if (cudaMemcpyAsync(&st, scratch, sizeof(int), cudaMemcpyDeviceToHost, stream) != cudaSuccess)
    return ZSA_ERR_CUDA;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return ZSA_ERR_CUDA;
  if (st == 0) return ZSA_OK;
  if (cudaMemsetAsync(scratch, 0, sizeof(int), stream) != cudaSuccess) return ZSA_ERR_CUDA;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return ZSA_ERR_CUDA;
  return ZSA_ERR_TIMEOUT;
}
