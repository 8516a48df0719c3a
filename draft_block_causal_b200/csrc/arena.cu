// arena.cu -- the weight arena and the opt-in L2 residency window.
//
// Every position of a draft block re-reads the head's matrices (W2 dominates: V x r), so the
// block's traffic is mostly re-reads of about 110 MB that B200's 126 MB L2 can hold.  Packing the
// matrices into one contiguous arena lets a single stream access-policy window cover them, so
// that the hardware keeps them in L2 (persisting hits) while base logits, hidden states and
// other streamed operands pass through (streaming misses).
#include "domino.h"
#include "internal.h"

#include <mutex>

namespace domino {
namespace {

inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

struct ArenaLayout {
  size_t W2, W1, W_hh, W_ih, b_ih, b_hh, hot_end, bytes;
};

// [W2][W1][W_hh][W_ih][b_ih][b_hh], each region 256-byte aligned: the matrices read at every
// position first, so that the hot range is one prefix of the arena.
ArenaLayout arena_layout(const domino_shape_t& s) {
  const size_t es = s.dtype == DOMINO_DTYPE_BF16 ? 2 : 4;
  ArenaLayout a{};
  size_t off = 0;
  auto take = [&](size_t elems) {
    const size_t o = off;
    off = align256(off + elems * es);
    return o;
  };
  a.W2 = take((size_t)s.V * s.r);
  a.W1 = take((size_t)s.r * (s.d + s.Hs));
  a.W_hh = take((size_t)3 * s.Hs * s.Hs);
  a.W_ih = take((size_t)3 * s.Hs * s.d);
  a.hot_end = off;
  a.b_ih = take((size_t)3 * s.Hs);
  a.b_hh = take((size_t)3 * s.Hs);
  a.bytes = off;
  return a;
}

std::mutex g_l2_mu;
// persisting set-aside of each device's context before the first window was set (-1: untouched)
long long g_saved_setaside[64];
bool g_saved_init = false;

}  // namespace
}  // namespace domino

using namespace domino;

extern "C" {

size_t domino_arena_bytes(const domino_shape_t* shape) {
  if (check_shape(shape) != DOMINO_OK) return 0;
  return arena_layout(*shape).bytes;
}

int domino_pack_weights(const domino_shape_t* shape, const domino_weights_t* src, void* arena, size_t arena_bytes,
                        domino_weights_t* packed, domino_stream_t stream) {
  int rc = check_shape(shape);
  if (rc != DOMINO_OK) return rc;
  if ((rc = check_weights(src)) != DOMINO_OK) return rc;
  if (!packed) return DOMINO_ERR_INVALID_ARGUMENT;
  const ArenaLayout a = arena_layout(*shape);
  if (!arena || (reinterpret_cast<uintptr_t>(arena) & 255u) || arena_bytes < a.bytes) return DOMINO_ERR_WORKSPACE;
  const domino_shape_t& s = *shape;
  const size_t es = s.dtype == DOMINO_DTYPE_BF16 ? 2 : 4;
  char* base = static_cast<char*>(arena);
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  struct Piece {
    const void* from;
    size_t at, elems;
  } pieces[] = {{src->W2, a.W2, (size_t)s.V * s.r},
                {src->W1, a.W1, (size_t)s.r * (s.d + s.Hs)},
                {src->W_hh, a.W_hh, (size_t)3 * s.Hs * s.Hs},
                {src->W_ih, a.W_ih, (size_t)3 * s.Hs * s.d},
                {src->b_ih, a.b_ih, (size_t)3 * s.Hs},
                {src->b_hh, a.b_hh, (size_t)3 * s.Hs}};
  for (const Piece& p : pieces)
    if (cudaMemcpyAsync(base + p.at, p.from, p.elems * es, cudaMemcpyDeviceToDevice, cs) != cudaSuccess)
      return DOMINO_ERR_CUDA;
  packed->embed = src->embed;
  packed->embed_proj = src->embed_proj;
  packed->W2 = base + a.W2;
  packed->W1 = base + a.W1;
  packed->W_hh = base + a.W_hh;
  packed->W_ih = base + a.W_ih;
  packed->b_ih = base + a.b_ih;
  packed->b_hh = base + a.b_hh;
  return DOMINO_OK;
}

int domino_set_l2_persistence(const domino_shape_t* shape, const domino_weights_t* weights, domino_stream_t stream,
                              float hit_ratio) {
  int rc = check_shape(shape);
  if (rc != DOMINO_OK) return rc;
  if ((rc = check_weights(weights)) != DOMINO_OK) return rc;
  if (!stream || !(hit_ratio >= 0.f && hit_ratio <= 1.f)) return DOMINO_ERR_INVALID_ARGUMENT;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return DOMINO_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_l2_mu);
  if (!g_saved_init) {
    for (long long& v : g_saved_setaside) v = -1;
    g_saved_init = true;
  }
  cudaStreamAttrValue attr = {};
  if (hit_ratio == 0.f) {  // clear: no window, persisting lines back to normal, set-aside restored
    attr.accessPolicyWindow.num_bytes = 0;
    if (cudaStreamSetAttribute(cs, cudaStreamAttributeAccessPolicyWindow, &attr) != cudaSuccess)
      return DOMINO_ERR_CUDA;
    if (cudaCtxResetPersistingL2Cache() != cudaSuccess) return DOMINO_ERR_CUDA;
    if (g_saved_setaside[dev] >= 0) {
      if (cudaDeviceSetLimit(cudaLimitPersistingL2CacheSize, (size_t)g_saved_setaside[dev]) != cudaSuccess)
        return DOMINO_ERR_CUDA;
      g_saved_setaside[dev] = -1;
    }
    return DOMINO_OK;
  }
  // the hot matrices must lie in one packed range (as domino_pack_weights lays them out)
  const domino_shape_t& s = *shape;
  const size_t es = s.dtype == DOMINO_DTYPE_BF16 ? 2 : 4;
  struct Range {
    const void* p;
    size_t bytes;
  } hot[] = {{weights->W2, (size_t)s.V * s.r * es},
             {weights->W1, (size_t)s.r * (s.d + s.Hs) * es},
             {weights->W_hh, (size_t)3 * s.Hs * s.Hs * es},
             {weights->W_ih, weights->embed_proj ? 0 : (size_t)3 * s.Hs * s.d * es}};
  uintptr_t lo = UINTPTR_MAX, hi = 0;
  size_t sum = 0;
  for (const Range& r : hot) {
    if (!r.bytes) continue;
    const uintptr_t b = reinterpret_cast<uintptr_t>(r.p);
    lo = b < lo ? b : lo;
    hi = b + r.bytes > hi ? b + r.bytes : hi;
    sum += r.bytes;
  }
  if (hi - lo > sum + 4096) return DOMINO_ERR_INVALID_ARGUMENT;  // not packed
  int max_persist = 0, max_window = 0;
  if (cudaDeviceGetAttribute(&max_persist, cudaDevAttrMaxPersistingL2CacheSize, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&max_window, cudaDevAttrMaxAccessPolicyWindowSize, dev) != cudaSuccess)
    return DOMINO_ERR_CUDA;
  if (max_persist <= 0 || max_window <= 0) return DOMINO_ERR_UNSUPPORTED;
  if (g_saved_setaside[dev] < 0) {
    size_t cur = 0;
    if (cudaDeviceGetLimit(&cur, cudaLimitPersistingL2CacheSize) != cudaSuccess) return DOMINO_ERR_CUDA;
    g_saved_setaside[dev] = (long long)cur;
  }
  const size_t span = hi - lo;
  const size_t setaside = span < (size_t)max_persist ? span : (size_t)max_persist;
  if (cudaDeviceSetLimit(cudaLimitPersistingL2CacheSize, setaside) != cudaSuccess) return DOMINO_ERR_CUDA;
  const size_t window = span < (size_t)max_window ? span : (size_t)max_window;
  // a window larger than the set-aside marks only that fraction of its lines persisting, so that
  // the persisting lines do not evict one another
  const double frac = (double)setaside / (double)window;
  attr.accessPolicyWindow.base_ptr = reinterpret_cast<void*>(lo);
  attr.accessPolicyWindow.num_bytes = window;
  attr.accessPolicyWindow.hitRatio = (float)(hit_ratio * (frac < 1.0 ? frac : 1.0));
  attr.accessPolicyWindow.hitProp = cudaAccessPropertyPersisting;
  attr.accessPolicyWindow.missProp = cudaAccessPropertyStreaming;
  if (cudaStreamSetAttribute(cs, cudaStreamAttributeAccessPolicyWindow, &attr) != cudaSuccess) return DOMINO_ERR_CUDA;
  return DOMINO_OK;
}

}  // extern "C"
