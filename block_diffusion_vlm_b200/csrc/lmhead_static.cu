// Fused LM head + confidence + commit with no caller-provided workspace.
//
// Some callers of this library cannot allocate device memory at the point
// where they call it: a serving process whose device memory is reserved up
// front by another framework's caching allocator, or an edge / robotics
// control loop that forbids cudaMalloc after start-up because an allocation
// can synchronise the whole device and stall the loop.  For them
// dvlm_lmhead_conf_commit_static keeps its scratch (split-tile partials,
// counters, per-CTA records, sums of squares) in one file-scope device array
// of fixed size.  The CUDA runtime creates the array on a GPU when it loads
// this library's device code there (with lazy loading, the default, at the
// first call that needs that code) and keeps it until the process exits or
// the device is reset.  The entry point allocates nothing and calls no
// allocating routine.
#include <cudaTypedefs.h>

#include <mutex>

#include "kernels.h"

namespace {

constexpr size_t kStaticScratchBytes = 6u << 20;  // 6 MiB
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_lm_scratch[kStaticScratchBytes];

std::mutex g_mu;
void* g_addr[kMaxDevices] = {};
unsigned long long g_ctx[kMaxDevices] = {};  // context the address belongs to

// Unique id of the current context (cuCtxGetId, fetched through the runtime
// so the library does not link libcuda); 0 when unavailable.
unsigned long long current_context_id() {
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  static PFN_cuCtxGetCurrent_v4000 get_cur = nullptr;
  static bool tried = false;
  if (!tried) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_cur = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    tried = true;
  }
  CUcontext c = nullptr;
  unsigned long long id = 0;
  if (!get_id || !get_cur || get_cur(&c) != CUDA_SUCCESS || !c || get_id(c, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// Device address of g_lm_scratch on the current device.  In host code the
// array's name is only a host-side stand-in, never a device address: the
// runtime returns the real one, looked up at set-up with that device current
// (the first call on the device), and that is what the kernels are given.
// A device reset gives the device a new context, in which the array may sit
// elsewhere: the address is looked up again when the current context is not
// the one it was taken in.
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  const unsigned long long ctx = current_context_id();
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_addr[dev] || ctx == 0 || g_ctx[dev] != ctx) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_lm_scratch);
    if (e != cudaSuccess) return e;
    g_addr[dev] = p;
    g_ctx[dev] = ctx;
  }
  *out = g_addr[dev];
  return cudaSuccess;
}

struct StaticLayout {
  size_t part, cnt, done, rec, ssq, bytes;
  size_t zero_begin, zero_end;  // counters that must start at zero
};

size_t up256(size_t v) { return (v + 255) / 256 * 256; }

StaticLayout layout(int NT, int P, int n_tiles, int H) {
  StaticLayout L{};
  size_t off = 0;
  L.part = off;
  off = up256(off + static_cast<size_t>(P) * NT * 128 * 4);
  L.cnt = off;
  L.zero_begin = off;
  off += static_cast<size_t>(n_tiles) * 4;
  L.done = off;
  off += 4;
  L.zero_end = off;
  off = up256(off);
  L.rec = off;
  off = up256(off + static_cast<size_t>(P) * NT * 16);
  L.ssq = off;
  off = up256(off + static_cast<size_t>(H / 128 + 1) * NT * 4);
  L.bytes = off;
  return L;
}

inline bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" dvlm_status dvlm_lmhead_conf_commit_static(
    const void* hidden, const void* w, int R, int H, int V, int apply_rmsnorm, float eps, uint8_t* masked,
    int32_t* tokens, float threshold, int32_t* top1_id, float* top1_prob, uint8_t* commit, int32_t* n_commit,
    const int32_t* anchor_id, const float* anchor_conf, int32_t* cert_len, int* dev_status, dvlm_stream stream) {
  using namespace dvlm;
  if (!hidden || !w) return DVLM_ERR_INVALID_ARG;
  if (R < 1 || R > 128 || H < 1 || V < 1) return DVLM_ERR_SHAPE;
  if (tokens && !masked) return DVLM_ERR_INVALID_ARG;
  const int nc = (anchor_id != nullptr) + (anchor_conf != nullptr) + (cert_len != nullptr);
  if (nc != 0 && nc != 3) return DVLM_ERR_INVALID_ARG;
  if (threshold != threshold) return DVLM_ERR_INVALID_ARG;
  if (apply_rmsnorm && !(eps > 0.f)) return DVLM_ERR_INVALID_ARG;
  if (H % 64 || (apply_rmsnorm && H % 128)) return DVLM_ERR_UNSUPPORTED;
  if (!al16(hidden) || !al16(w)) return DVLM_ERR_INVALID_ARG;
  // Sizes beyond the fixed scratch are refused, never truncated.
  if (R > 32) return DVLM_ERR_WORKSPACE;
  const int P = device_sm_count();
  if (P <= 0) return DVLM_ERR_CUDA;
  const int NT = R <= 16 ? 16 : 32;
  const int n_tiles = (V + 127) / 128;
  const StaticLayout lay = layout(NT, P, n_tiles, H);
  if (lay.bytes > kStaticScratchBytes) return DVLM_ERR_WORKSPACE;

  void* base = nullptr;
  if (scratch_address(&base) != cudaSuccess) return DVLM_ERR_CUDA;
  uint8_t* s = static_cast<uint8_t*>(base);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // The array keeps the previous call's contents: the counters that the
  // kernel expects at zero are cleared on the stream before each launch.
  if (cudaMemsetAsync(s + lay.zero_begin, 0, lay.zero_end - lay.zero_begin, st) != cudaSuccess)
    return DVLM_ERR_CUDA;

  CUtensorMap mw, mh;
  bool ok = make_tmap_2d(&mw, w, H, V, static_cast<uint64_t>(H) * 2, 64, 128);
  ok &= make_tmap_2d(&mh, hidden, H, R, static_cast<uint64_t>(H) * 2, 64, NT);
  if (!ok) return DVLM_ERR_CUDA;
  LmArgs a{};
  a.R = R;
  a.V = V;
  a.part = reinterpret_cast<float*>(s + lay.part);
  a.cnt = reinterpret_cast<int*>(s + lay.cnt);
  a.rec = reinterpret_cast<float*>(s + lay.rec);
  a.done = reinterpret_cast<int*>(s + lay.done);
  a.masked = masked;
  a.tokens = tokens;
  a.threshold = threshold;
  a.top1_id = top1_id;
  a.top1_prob = top1_prob;
  a.commit = commit;
  a.n_commit = n_commit;
  a.anchor_id = anchor_id;
  a.anchor_conf = anchor_conf;
  a.cert_len = cert_len;
  a.status = dev_status;
  if (apply_rmsnorm) {
    float* ssq = reinterpret_cast<float*>(s + lay.ssq);
    if (launch_embed_bf16(nullptr, static_cast<const bf16*>(hidden), R, nullptr, nullptr, 0, R, H, V, nullptr, ssq,
                          NT, dev_status, false, st) != cudaSuccess)
      return DVLM_ERR_CUDA;
    a.ssq_in = ssq;
    a.n_ssq = H / 128;
    a.inv_h = 1.0f / H;
    a.eps = eps;
  }
  const long long units = static_cast<long long>(n_tiles) * (H / 64);
  const int Pl = static_cast<int>(units < P ? units : P);
  return launch_lmhead(NT, mw, mh, n_tiles, H / 64, Pl, a, false, st) == cudaSuccess ? DVLM_OK : DVLM_ERR_CUDA;
}
