// noalloc.cu -- greedy drafting with library-owned scratch, for callers that cannot allocate.
//
// domino_draft_greedy needs a caller-provided workspace.  Some callers cannot provide one at
// the point of the call: a serving process that carved all free device memory into its weight
// and KV-cache pools at start-up (a late cudaMalloc fails or fragments those pools), a plugin
// running inside a host runtime that owns the device allocator and forbids allocations of its
// own, or a latency-critical loop that must not pay the implicit synchronisation and
// unpredictable cost of an allocation.  This entry point takes no workspace: its scratch is a
// fixed, file-scope device array that every GPU which loads the library holds until the
// process exits.
#include "domino.h"
#include "internal.h"
#include "persistent.h"

#include <mutex>

namespace domino {
namespace {

// Scratch of the fused greedy kernel: status word, barrier counter, argmax keys, the W1
// accumulators, the H-projections and the state ping-pong.  DOMINO_NOALLOC_SCRATCH_BYTES bytes
// per device.
static __device__ __align__(256) unsigned char g_noalloc_scratch[DOMINO_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices] = {};
std::mutex g_scratch_mu;

inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// The regions the fused kernel touches, packed from `base`.  sync, keys and a_acc stay adjacent
// and in this order: the launcher clears them with one memset on every call.
Workspace compact_layout(const Shape& s, void* base) {
  Workspace w{};
  char* p = static_cast<char*>(base);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = align256(off + bytes);
    return p ? p + o : nullptr;
  };
  const size_t BL = (size_t)s.B * s.L;
  w.status = reinterpret_cast<int32_t*>(take(sizeof(int32_t)));
  w.sync = reinterpret_cast<uint32_t*>(take(kSyncWords * sizeof(uint32_t)));
  w.keys = reinterpret_cast<uint64_t*>(take(BL * sizeof(uint64_t)));
  w.a_acc = reinterpret_cast<unsigned long long*>(take(acc_bytes(s.B, s.r)));
  w.P = reinterpret_cast<float*>(take(BL * s.r * sizeof(float)));
  w.S = reinterpret_cast<float*>(take(2 * (size_t)s.B * s.Hs * sizeof(float)));
  w.bytes = off;
  return w;
}

// Device address of the scratch array on the current device, looked up once per device.  A
// host-side reference to g_noalloc_scratch names a host shadow, not device memory, so the
// address must come from cudaGetSymbolAddress with the device current.
cudaError_t scratch_on_current_device(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = ptr;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace domino

using namespace domino;

extern "C" int domino_draft_greedy_noalloc(const domino_shape_t* shape, const domino_weights_t* w,
                                           const void* base_logits, const void* hidden, const float* S0,
                                           int32_t* tokens_out, float* logits_out, float* states_out,
                                           int32_t* status_dev, domino_stream_t stream) {
  auto a16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
  int rc = check_shape(shape);
  if (rc != DOMINO_OK) return rc;
  // the same weight checks as domino_draft_greedy, the optional projection table included
  if ((rc = check_weights(w)) != DOMINO_OK) return rc;
  if (!base_logits || !hidden || !S0 || !tokens_out) return DOMINO_ERR_INVALID_ARGUMENT;
  if (!a16(base_logits) || !a16(hidden) || !a16(S0) || !a16(tokens_out) || (logits_out && !a16(logits_out)) ||
      (states_out && !a16(states_out)))
    return DOMINO_ERR_INVALID_ARGUMENT;
  const Shape s{shape->B, shape->L, shape->d, shape->Hs, shape->r, shape->V, shape->dtype};
  if (!use_persistent_greedy(s)) return DOMINO_ERR_UNSUPPORTED;
  if (compact_layout(s, nullptr).bytes > DOMINO_NOALLOC_SCRATCH_BYTES) return DOMINO_ERR_SCRATCH_LIMIT;
  void* base = nullptr;
  if (scratch_on_current_device(&base) != cudaSuccess) return DOMINO_ERR_CUDA;
  const Workspace ws = compact_layout(s, base);
  int32_t* st = status_dev ? status_dev : ws.status;
  cudaError_t e = launch_persistent_greedy(s, *w, base_logits, hidden, S0, tokens_out, logits_out, states_out, ws,
                                           st, spin_limit(), static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? DOMINO_OK : DOMINO_ERR_CUDA;
}
