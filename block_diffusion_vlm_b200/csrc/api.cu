// C ABI of the library (declared in include/dvlm.h).  Every entry point
// validates its arguments on the host and returns an error status before
// launching anything; kernels report device-side problems through the
// caller's status word.
#include <cmath>
#include <cstdlib>
#include <new>

#include "engine.h"

using namespace dvlm;

namespace dvlm {
cudaError_t engine_forward(dvlm_engine* e, const FwdSpec& f, cudaStream_t s);
cudaError_t engine_step(dvlm_engine* e, const dvlm_decode_cfg& cfg, int max_new, int n_out_host, int* emitted,
                        dvlm_stats* st, cudaStream_t s);
cudaError_t engine_collect_stats(dvlm_engine* e, dvlm_stats* st, cudaStream_t s);
size_t engine_workspace_bytes(dvlm_engine* e, int P);
size_t engine_carve(dvlm_engine* e, void* ws, int P);
bool engine_build_maps(dvlm_engine* e);
void engine_plan(dvlm_engine* e);
cudaError_t engine_profile(dvlm_engine* e, const FwdSpec& f0, float* ms, int* counts, cudaStream_t s);
dvlm_status engine_set_option(dvlm_engine* e, const char* name, int v);
int engine_get_option(dvlm_engine* e, const char* name);
void engine_set_trace(dvlm_engine* e, void* buf, int cap, int32_t* cnt);
bool prefill_gemm_supported(const dvlm_engine* e);
bool quad_supported(const dvlm_engine* e, int B);
cudaError_t engine_forward_quad(dvlm_engine* e, const int32_t* draft, int B, void* x_out, cudaStream_t s);
bool engine_set_paged(dvlm_engine* e, void* k_pages, void* v_pages, const int32_t* table, int n_pages,
                      int max_pages);
cudaError_t engine_prefill_gemm(dvlm_engine* e, const void* vision, int n_vis, const int32_t* ids, int n_ids,
                                cudaStream_t s);
cudaError_t launch_topk_commit(const float* p1, const int32_t* ids, const int32_t* other_ids, uint8_t* masked,
                               int32_t* tokens, int R, int k, uint8_t* commit, int32_t* n_commit, cudaStream_t s);
}  // namespace dvlm

namespace {

constexpr int kDefaultSms = 148;

inline bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline cudaStream_t cs(dvlm_stream s) { return static_cast<cudaStream_t>(s); }
inline dvlm_status cuda_status(cudaError_t e) { return e == cudaSuccess ? DVLM_OK : DVLM_ERR_CUDA; }
inline int sms_or_default() {
  const int n = device_sm_count();
  return n > 0 ? n : kDefaultSms;
}
// Attention cluster size for the current device: 16 CTAs where two such
// clusters can be resident at once, else 8 (queried once per device).
inline int attn_cluster_for_device() {
  static int cached[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return attn_split_cl_max_clusters(16) >= 2 ? 16 : 8;
  if (cached[dev] == 0) cached[dev] = attn_split_cl_max_clusters(16) >= 2 ? 16 : 8;
  return cached[dev];
}
inline int lm_nt(int R) { return R <= 16 ? 16 : R <= 32 ? 32 : R <= 64 ? 64 : 128; }

struct LmWs {
  float* part;
  int* cnt;
  float* rec;
  int* done;
  float* ssq;
  float* p1;
  int32_t* ids;
  size_t bytes;
};

LmWs carve_lm(uint8_t* base, int R, int V, int H, dvlm_dtype dt, int P) {
  LmWs w{};
  size_t off = 0;
  auto take = [&](size_t n) {
    off = (off + 255) / 256 * 256;
    uint8_t* p = base ? base + off : nullptr;
    off += n;
    return p;
  };
  if (dt == DVLM_BF16) {
    const int NT = lm_nt(R);
    const int n_tiles = (V + 127) / 128;
    w.part = reinterpret_cast<float*>(take(static_cast<size_t>(P) * NT * 128 * 4));
    w.cnt = reinterpret_cast<int*>(take(static_cast<size_t>(n_tiles) * 4));
    w.rec = reinterpret_cast<float*>(take(static_cast<size_t>(P) * NT * 16));
    w.done = reinterpret_cast<int*>(take(4));
    w.ssq = reinterpret_cast<float*>(take(static_cast<size_t>(H / 128 + 1) * NT * 4));
  } else {
    w.ssq = reinterpret_cast<float*>(take(static_cast<size_t>(R) * 4));
    w.p1 = reinterpret_cast<float*>(take(static_cast<size_t>(R) * 4));
    w.ids = reinterpret_cast<int32_t*>(take(static_cast<size_t>(R) * 4));
  }
  w.bytes = (off + 255) / 256 * 256;
  return w;
}

inline int spec_splits(int b, int B) {
  const int rows = b * B;
  int s = (2 * kDefaultSms + rows - 1) / rows;
  return s < 1 ? 1 : (s > 64 ? 64 : s);
}

bool model_ok(const dvlm_model* m) {
  if (!m || m->n_layers < 1 || m->hidden < 1 || m->n_q_heads < 1 || m->n_kv_heads < 1 || m->head_dim < 2 ||
      m->inter < 1 || m->vocab < 1)
    return false;
  if (m->n_q_heads % m->n_kv_heads || m->head_dim % 2) return false;
  if (m->mask_id < 0 || m->mask_id >= m->vocab) return false;
  if (!(m->eps > 0.f) || !(m->rope_base > 0.f)) return false;
  if (m->dtype != DVLM_BF16 && m->dtype != DVLM_FP32 && m->dtype != DVLM_FP8_W8A8) return false;
  if (m->dtype == DVLM_FP8_W8A8 && !(m->sqkv && m->so && m->sgate && m->sup && m->sdown)) return false;
  return m->embed && m->wqkv && m->wo && m->wgate && m->wup && m->wdown && m->lm_head;
}

dvlm_status bf16_model_supported(const dvlm_model* m) {
  if (m->head_dim != 128 || m->n_q_heads != 8 * m->n_kv_heads || m->hidden % 128 || m->inter % 64 ||
      (m->n_q_heads * m->head_dim) % 128)
    return DVLM_ERR_UNSUPPORTED;
  const void* p[] = {m->embed, m->wqkv, m->wo, m->wgate, m->wup, m->wdown, m->lm_head};
  for (const void* q : p)
    if (!al16(q)) return DVLM_ERR_INVALID_ARG;
  // W8A8: 128-wide k blocks of E4M3 codes in every projection
  if (m->dtype == DVLM_FP8_W8A8 && (m->inter % 128 || (m->n_q_heads * m->head_dim) % 128 || m->hidden % 128))
    return DVLM_ERR_UNSUPPORTED;
  return DVLM_OK;
}

}  // namespace

extern "C" {

const char* dvlm_status_string(int status) {
  switch (status) {
    case DVLM_OK: return "ok";
    case DVLM_ERR_INVALID_ARG: return "invalid argument";
    case DVLM_ERR_SHAPE: return "bad shape";
    case DVLM_ERR_UNSUPPORTED: return "unsupported";
    case DVLM_ERR_CACHE_OVERFLOW: return "KV cache overflow";
    case DVLM_ERR_TIMEOUT: return "device wait timed out";
    case DVLM_ERR_CUDA: return "CUDA error";
    case DVLM_ERR_WORKSPACE: return "workspace too small";
    case DVLM_ERR_BOUNDS: return "index out of bounds";
  }
  return "unknown status";
}

int dvlm_version(void) { return 100; }

int dvlm_device_sm_count(void) { return device_sm_count(); }

// ------------------------------------------------------------ attention
dvlm_status dvlm_block_attn(const void* q, void* out, const void* k_cache, const void* v_cache, int n_batch,
                            int n_rows, int n_clean, int L, int Lmax, int Hq, int Hkv, int D, float scale,
                            dvlm_dtype dt, int* dev_status, dvlm_stream stream) {
  if (!q || !out || !k_cache || !v_cache) return DVLM_ERR_INVALID_ARG;
  if (dt != DVLM_BF16 && dt != DVLM_FP32) return DVLM_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return DVLM_ERR_INVALID_ARG;
  if (n_batch < 1 || n_rows < 1 || n_clean < 0 || n_clean > n_rows || L < 0 || Lmax < 1 || Hq < 1 || Hkv < 1 ||
      D < 1 || Hq % Hkv)
    return DVLM_ERR_SHAPE;
  if (static_cast<long long>(L) + n_rows > Lmax) return DVLM_ERR_CACHE_OVERFLOW;
  if (dt == DVLM_FP32) {
    if (D > 128) return DVLM_ERR_UNSUPPORTED;
    return cuda_status(f32_attention(static_cast<const float*>(q), static_cast<float*>(out),
                                     static_cast<const float*>(k_cache), static_cast<const float*>(v_cache), n_batch,
                                     n_rows, n_clean, L, nullptr, Lmax, Hq, Hkv, D, scale, cs(stream)));
  }
  if (D != 128 || Hq != 8 * Hkv) return DVLM_ERR_UNSUPPORTED;
  if (Lmax % 8) return DVLM_ERR_SHAPE;
  if (!al16(q) || !al16(out) || !al16(k_cache) || !al16(v_cache)) return DVLM_ERR_INVALID_ARG;
  const int n_groups = (n_rows + 15) / 16;
  if (static_cast<long long>(n_batch) * n_groups > 65535) return DVLM_ERR_SHAPE;
  CUtensorMap mq, mk, mv;
  const uint64_t rows_total = static_cast<uint64_t>(n_batch) * n_rows;
  bool ok = make_tmap_3d(&mq, q, D, Hq, rows_total, D * 2, static_cast<uint64_t>(Hq) * D * 2, 64, 8, 16);
  ok &= make_tmap_2d(&mk, k_cache, D, static_cast<uint64_t>(n_batch) * Hkv * Lmax, D * 2, 64, 64);
  ok &= make_tmap_2d(&mv, v_cache, Lmax, static_cast<uint64_t>(n_batch) * Hkv * D, static_cast<uint64_t>(Lmax) * 2,
                     64, 128);
  if (!ok) return DVLM_ERR_CUDA;
  AttnArgs a{};
  a.n_rows = n_rows;
  a.n_clean = n_clean;
  a.n_batch = n_batch;
  a.L_static = L;
  a.d_len = nullptr;
  a.Lmax = Lmax;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.kv_base = 0;
  a.scale_log2 = static_cast<float>(scale * 1.4426950408889634);
  a.out = static_cast<bf16*>(out);
  a.status = dev_status;
  return cuda_status(launch_attn_split_cl(mq, mk, mv, a, attn_cluster_for_device(), false, cs(stream)));
}

size_t dvlm_block_attn_split_workspace_size(int n_batch, int n_rows, int Hkv, int splits) {
  if (n_batch < 1 || n_rows < 1 || Hkv < 1 || splits < 1 || splits > 64) return 0;
  return attn_split_scratch_bytes(n_batch * ((n_rows + 15) / 16) * Hkv, splits);
}

dvlm_status dvlm_block_attn_split(const void* q, void* out, const void* k_cache, const void* v_cache, int n_batch,
                                  int n_rows, int n_clean, int L, int Lmax, int Hq, int Hkv, int D, float scale,
                                  int splits, void* workspace, size_t ws_bytes, int* dev_status,
                                  dvlm_stream stream) {
  if (!q || !out || !k_cache || !v_cache) return DVLM_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return DVLM_ERR_INVALID_ARG;
  if (n_batch < 1 || n_rows < 1 || n_clean < 0 || n_clean > n_rows || L < 0 || Lmax < 1 || Hq < 1 || Hkv < 1 ||
      D < 1 || Hq % Hkv || splits < 1 || splits > 64)
    return DVLM_ERR_SHAPE;
  if (static_cast<long long>(L) + n_rows > Lmax) return DVLM_ERR_CACHE_OVERFLOW;
  if (D != 128 || Hq != 8 * Hkv) return DVLM_ERR_UNSUPPORTED;
  if (Lmax % 8) return DVLM_ERR_SHAPE;
  if (!al16(q) || !al16(out) || !al16(k_cache) || !al16(v_cache) || !al16(workspace)) return DVLM_ERR_INVALID_ARG;
  const int n_groups = (n_rows + 15) / 16;
  if (static_cast<long long>(n_batch) * n_groups > 65535) return DVLM_ERR_SHAPE;
  if (!workspace || ws_bytes < attn_split_scratch_bytes(n_batch * n_groups * Hkv, splits)) return DVLM_ERR_WORKSPACE;
  CUtensorMap mq, mk, mv;
  const uint64_t rows_total = static_cast<uint64_t>(n_batch) * n_rows;
  bool ok = make_tmap_3d(&mq, q, D, Hq, rows_total, D * 2, static_cast<uint64_t>(Hq) * D * 2, 64, 8, 16);
  ok &= make_tmap_2d(&mk, k_cache, D, static_cast<uint64_t>(n_batch) * Hkv * Lmax, D * 2, 64, 64);
  ok &= make_tmap_2d(&mv, v_cache, Lmax, static_cast<uint64_t>(n_batch) * Hkv * D, static_cast<uint64_t>(Lmax) * 2,
                     64, 128);
  if (!ok) return DVLM_ERR_CUDA;
  AttnArgs a{};
  a.n_rows = n_rows;
  a.n_clean = n_clean;
  a.n_batch = n_batch;
  a.L_static = L;
  a.Lmax = Lmax;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.scale_log2 = static_cast<float>(scale * 1.4426950408889634);
  a.out = static_cast<bf16*>(out);
  a.status = dev_status;
  return cuda_status(launch_attn_split(mq, mk, mv, a, splits, workspace, false, cs(stream)));
}

dvlm_status dvlm_block_attn_paged(const void* q, void* out, const void* k_pages, const void* v_pages,
                                  const int32_t* block_table, const int32_t* lens, int n_batch, int n_rows,
                                  int n_clean, int n_pages, int max_pages, int Hq, int Hkv, int D, float scale,
                                  int* dev_status, dvlm_stream stream) {
  if (!q || !out || !k_pages || !v_pages || !block_table || !lens) return DVLM_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return DVLM_ERR_INVALID_ARG;
  if (n_batch < 1 || n_rows < 1 || n_rows > 64 || n_clean < 0 || n_clean > n_rows || n_pages < 1 || max_pages < 1 ||
      Hq < 1 || Hkv < 1 || D < 1 || Hq % Hkv)
    return DVLM_ERR_SHAPE;
  if (D != 128 || Hq != 8 * Hkv) return DVLM_ERR_UNSUPPORTED;
  if (!al16(q) || !al16(out) || !al16(k_pages) || !al16(v_pages)) return DVLM_ERR_INVALID_ARG;
  const int n_groups = (n_rows + 15) / 16;
  if (static_cast<long long>(n_batch) * n_groups > 65535) return DVLM_ERR_SHAPE;
  CUtensorMap mq, mk, mv;
  const uint64_t rows_total = static_cast<uint64_t>(n_batch) * n_rows;
  const uint64_t page_rows = static_cast<uint64_t>(n_pages) * Hkv;
  bool ok = make_tmap_3d(&mq, q, D, Hq, rows_total, D * 2, static_cast<uint64_t>(Hq) * D * 2, 64, 8, 16);
  ok &= make_tmap_2d(&mk, k_pages, D, page_rows * 64, D * 2, 64, 64);
  ok &= make_tmap_2d(&mv, v_pages, 64, page_rows * D, 64 * 2, 64, 128);
  if (!ok) return DVLM_ERR_CUDA;
  AttnArgs a{};
  a.n_rows = n_rows;
  a.n_clean = n_clean;
  a.n_batch = n_batch;
  a.Lmax = 64;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.kv_base = 0;
  a.scale_log2 = static_cast<float>(scale * 1.4426950408889634);
  a.out = static_cast<bf16*>(out);
  a.status = dev_status;
  a.block_table = block_table;
  a.max_pages = max_pages;
  a.n_pages = n_pages;
  a.d_lens = lens;
  return cuda_status(launch_attn_split_cl(mq, mk, mv, a, attn_cluster_for_device(), false, cs(stream)));
}

// ------------------------------------------------------------ LM head
size_t dvlm_lmhead_workspace_size(int R, int V, int H, dvlm_dtype dt) {
  if (R < 1 || R > 128 || V < 1 || H < 1) return 0;
  return carve_lm(nullptr, R, V, H, dt, sms_or_default()).bytes;
}

dvlm_status dvlm_lmhead_conf_commit(const void* hidden, const void* w, int R, int H, int V, dvlm_dtype dt,
                                    int apply_rmsnorm, float eps, uint8_t* masked, int32_t* tokens, float threshold,
                                    int32_t* top1_id, float* top1_prob, uint8_t* commit, int32_t* n_commit,
                                    const int32_t* anchor_id, const float* anchor_conf, int32_t* cert_len,
                                    void* workspace, size_t ws_bytes, int* dev_status, dvlm_stream stream) {
  if (!hidden || !w) return DVLM_ERR_INVALID_ARG;
  if (dt != DVLM_BF16 && dt != DVLM_FP32) return DVLM_ERR_INVALID_ARG;
  if (R < 1 || R > 128 || H < 1 || V < 1) return DVLM_ERR_SHAPE;
  if (tokens && !masked) return DVLM_ERR_INVALID_ARG;
  const int nc = (anchor_id != nullptr) + (anchor_conf != nullptr) + (cert_len != nullptr);
  if (nc != 0 && nc != 3) return DVLM_ERR_INVALID_ARG;
  if (std::isnan(threshold)) return DVLM_ERR_INVALID_ARG;
  if (apply_rmsnorm && !(eps > 0.f)) return DVLM_ERR_INVALID_ARG;
  const int P = sms_or_default();
  LmWs lw = carve_lm(nullptr, R, V, H, dt, P);
  if (!workspace) return DVLM_ERR_WORKSPACE;
  if (ws_bytes < lw.bytes) return DVLM_ERR_WORKSPACE;
  if (!al16(workspace)) return DVLM_ERR_INVALID_ARG;
  lw = carve_lm(static_cast<uint8_t*>(workspace), R, V, H, dt, P);
  LmArgs a{};
  a.R = R;
  a.V = V;
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
  if (dt == DVLM_FP32) {
    cudaError_t e = cudaSuccess;
    if (apply_rmsnorm) e = f32_rowscale(static_cast<const float*>(hidden), H, R, H, eps, lw.ssq, cs(stream));
    if (e != cudaSuccess) return DVLM_ERR_CUDA;
    return cuda_status(f32_lmhead(static_cast<const float*>(hidden), static_cast<const float*>(w), R, H, V,
                                  apply_rmsnorm ? lw.ssq : nullptr, lw.p1, lw.ids, a, cs(stream)));
  }
  if (H % 128 && apply_rmsnorm) return DVLM_ERR_UNSUPPORTED;
  if (H % 64) return DVLM_ERR_UNSUPPORTED;
  if (!al16(hidden) || !al16(w)) return DVLM_ERR_INVALID_ARG;
  const int NT = lm_nt(R);
  CUtensorMap mw, mh;
  bool ok = make_tmap_2d(&mw, w, H, V, static_cast<uint64_t>(H) * 2, 64, 128);
  ok &= make_tmap_2d(&mh, hidden, H, R, static_cast<uint64_t>(H) * 2, 64, NT);
  if (!ok) return DVLM_ERR_CUDA;
  a.part = lw.part;
  a.cnt = lw.cnt;
  a.rec = lw.rec;
  a.done = lw.done;
  if (apply_rmsnorm) {
    cudaError_t e = launch_embed_bf16(nullptr, static_cast<const bf16*>(hidden), R, nullptr, nullptr, 0, R, H, V,
                                      nullptr, lw.ssq, NT, dev_status, false, cs(stream));
    if (e != cudaSuccess) return DVLM_ERR_CUDA;
    a.ssq_in = lw.ssq;
    a.n_ssq = H / 128;
    a.inv_h = 1.0f / H;
    a.eps = eps;
  }
  const int n_tiles = (V + 127) / 128;
  const long long units = static_cast<long long>(n_tiles) * (H / 64);
  const int Pl = static_cast<int>(units < P ? units : P);
  return cuda_status(launch_lmhead(NT, mw, mh, n_tiles, H / 64, Pl, a, false, cs(stream)));
}

// ------------------------------------------------------------ speculative accept
size_t dvlm_spec_workspace_size(int b, int B, int V) {
  if (b < 1 || B < 1 || V < 1) return 0;
  const size_t part = static_cast<size_t>(b) * B * spec_splits(b, B) * 2 * 4;
  return (part + 255) / 256 * 256 + static_cast<size_t>(b) * 4 + 256;
}

dvlm_status dvlm_topk_commit(const float* top1_prob, const int32_t* top1_id, uint8_t* masked, int32_t* tokens,
                             int R, int k, uint8_t* commit, int32_t* n_commit, int* dev_status, dvlm_stream stream) {
  (void)dev_status;
  if (!top1_prob || !top1_id || !masked || !tokens) return DVLM_ERR_INVALID_ARG;
  if (R < 1 || R > 128 || k < 0) return DVLM_ERR_SHAPE;
  return cuda_status(
      launch_topk_commit(top1_prob, top1_id, nullptr, masked, tokens, R, k, commit, n_commit, cs(stream)));
}

dvlm_status dvlm_divergence_first_commit(const float* full_prob, const int32_t* full_id, const int32_t* text_id,
                                         uint8_t* masked, int32_t* tokens, int R, int k, uint8_t* commit,
                                         int32_t* n_commit, int* dev_status, dvlm_stream stream) {
  (void)dev_status;
  if (!full_prob || !full_id || !text_id || !masked || !tokens) return DVLM_ERR_INVALID_ARG;
  if (R < 1 || R > 128 || k < 0) return DVLM_ERR_SHAPE;
  return cuda_status(
      launch_topk_commit(full_prob, full_id, text_id, masked, tokens, R, k, commit, n_commit, cs(stream)));
}

dvlm_status dvlm_spec_verify_accept(const void* verify_logits, const int32_t* verify_ids, const int32_t* draft_ids,
                                    int b, int B, int V, int32_t* accept_len, int32_t* cache_len, int poison_tail,
                                    void* k_cache, void* v_cache, int n_layers, int Hkv, int D, int Lmax,
                                    void* workspace, size_t ws_bytes, int* dev_status, dvlm_stream stream) {
  if (!draft_ids || !accept_len) return DVLM_ERR_INVALID_ARG;
  if (!verify_logits && !verify_ids) return DVLM_ERR_INVALID_ARG;
  if (b < 1 || B < 1 || B > 64 || V < 1) return DVLM_ERR_SHAPE;
  if (poison_tail) {
    if (!cache_len || !k_cache || !v_cache) return DVLM_ERR_INVALID_ARG;
    if (n_layers < 1 || Hkv < 1 || D < 1 || Lmax < 1) return DVLM_ERR_SHAPE;
  }
  bf16* kc = static_cast<bf16*>(k_cache);
  bf16* vc = static_cast<bf16*>(v_cache);
  if (verify_logits) {
    const size_t need = dvlm_spec_workspace_size(b, B, V);
    if (!workspace || ws_bytes < need) return DVLM_ERR_WORKSPACE;
    if (!al16(verify_logits) || !al16(workspace)) return DVLM_ERR_INVALID_ARG;
    const int splits = spec_splits(b, B);
    const size_t part = (static_cast<size_t>(b) * B * splits * 2 * 4 + 255) / 256 * 256;
    float* ws_part = static_cast<float*>(workspace);
    int* ws_cnt = reinterpret_cast<int*>(static_cast<uint8_t*>(workspace) + part);
    return cuda_status(launch_spec_logits(static_cast<const bf16*>(verify_logits), draft_ids, b, B, V, accept_len,
                                          cache_len, poison_tail, kc, vc, n_layers, Hkv, D, Lmax, ws_part, ws_cnt,
                                          splits, dev_status, cs(stream)));
  }
  return cuda_status(launch_spec_ids(verify_ids, draft_ids, b, B, accept_len, cache_len, poison_tail, kc, vc,
                                     n_layers, Hkv, D, Lmax, dev_status, cs(stream)));
}

// ------------------------------------------------------------ FP8 weights
dvlm_status dvlm_quantize_rows_e4m3(const void* a, int rows, int K, uint8_t* codes, float* scales,
                                    dvlm_stream stream) {
  if (!a || !codes || !scales) return DVLM_ERR_INVALID_ARG;
  if (rows < 1 || K < 1) return DVLM_ERR_SHAPE;
  return cuda_status(launch_quantize_rows_e4m3(static_cast<const bf16*>(a), rows, K, codes, scales, cs(stream)));
}

// ------------------------------------------------------------ engine
size_t dvlm_engine_workspace_size(const dvlm_model* m, int Lmax, int max_block, int max_ctx) {
  if (!model_ok(m) || Lmax < 1 || max_block < 1 || max_block > kNT || max_ctx < 0) return 0;
  dvlm_engine tmp;
  tmp.m = *m;
  tmp.bf16 = m->dtype != DVLM_FP32;
  tmp.fp8 = m->dtype == DVLM_FP8_W8A8;
  tmp.Lmax = Lmax;
  tmp.max_block = max_block;
  tmp.max_ctx = max_ctx;
  return engine_workspace_bytes(&tmp, sms_or_default());
}

dvlm_status dvlm_engine_create(const dvlm_model* m, void* k_cache, void* v_cache, int Lmax, int max_block,
                               int max_ctx, void* workspace, size_t ws_bytes, dvlm_stream stream, dvlm_engine** out) {
  if (!out) return DVLM_ERR_INVALID_ARG;
  *out = nullptr;
  if (!model_ok(m) || !k_cache || !v_cache) return DVLM_ERR_INVALID_ARG;
  if (Lmax < 1 || max_block < 1 || max_block > kNT || max_ctx < 0) return DVLM_ERR_SHAPE;
  if (m->dtype != DVLM_FP32) {
    const dvlm_status st = bf16_model_supported(m);
    if (st != DVLM_OK) return st;
    if (Lmax % 8 || !al16(k_cache) || !al16(v_cache)) return DVLM_ERR_INVALID_ARG;
  } else if (m->head_dim > 128) {
    return DVLM_ERR_UNSUPPORTED;
  }
  if (!workspace || !al16(workspace)) return DVLM_ERR_WORKSPACE;
  const int sm = device_sm_count();
  if (sm <= 0) return DVLM_ERR_CUDA;
  dvlm_engine* e = new (std::nothrow) dvlm_engine();
  if (!e) return DVLM_ERR_CUDA;
  e->m = *m;
  e->bf16 = m->dtype != DVLM_FP32;
  e->fp8 = m->dtype == DVLM_FP8_W8A8;
  e->Lmax = Lmax;
  e->max_block = max_block;
  e->max_ctx = max_ctx;
  e->kc = k_cache;
  e->vc = v_cache;
  e->sm = sm;
  const size_t need = engine_workspace_bytes(e, sm);
  if (ws_bytes < need) {
    delete e;
    return DVLM_ERR_WORKSPACE;
  }
  engine_carve(e, workspace, sm);
  if (cudaMemsetAsync(workspace, 0, need, cs(stream)) != cudaSuccess) {
    delete e;
    return DVLM_ERR_CUDA;
  }
  if (e->bf16 && !engine_build_maps(e)) {
    delete e;
    return DVLM_ERR_CUDA;
  }
  engine_plan(e);
  *out = e;
  return DVLM_OK;
}

dvlm_status dvlm_engine_destroy(dvlm_engine* e) {
  if (!e) return DVLM_ERR_INVALID_ARG;
  for (auto& kv : e->graphs) cudaGraphExecDestroy(kv.second);
  delete e;
  return DVLM_OK;
}

dvlm_status dvlm_prefill(dvlm_engine* e, const void* vision, int n_vision, const int32_t* ids, int n_ids,
                         dvlm_stream stream) {
  if (!e) return DVLM_ERR_INVALID_ARG;
  if (n_vision < 0 || n_ids < 0 || n_vision + n_ids < 1) return DVLM_ERR_SHAPE;
  if ((n_vision > 0 && !vision) || (n_ids > 0 && !ids)) return DVLM_ERR_INVALID_ARG;
  if (n_vision + n_ids > e->Lmax) return DVLM_ERR_CACHE_OVERFLOW;
  if (e->bf16 && n_vision > 0 && !al16(vision)) return DVLM_ERR_INVALID_ARG;
  cudaStream_t s = cs(stream);
  const int n_ctx = n_vision + n_ids;
  e->quad_ready = false;
  if (e->prefill_gemm && n_ctx <= e->max_ctx && prefill_gemm_supported(e))
    return cuda_status(engine_prefill_gemm(e, vision, n_vision, ids, n_ids, s));
  if (cudaMemsetAsync(e->d_len, 0, 4, s) != cudaSuccess) return DVLM_ERR_CUDA;
  const size_t es = e->bf16 ? 2 : 4;
  for (int c0 = 0; c0 < n_ctx; c0 += kNT) {
    const int n = std::min(kNT, n_ctx - c0);
    FwdSpec f;
    f.n_src = std::max(0, std::min(n, n_vision - c0));
    f.rows_in = f.n_src > 0 ? static_cast<const uint8_t*>(vision) + static_cast<size_t>(c0) * e->m.hidden * es
                            : nullptr;
    f.tokens = ids ? ids + std::max(0, c0 - n_vision) : nullptr;
    f.n_rows = n;
    f.n_clean = n;
    f.advance = true;
    f.lm = (c0 + n == n_ctx);
    if (f.lm) {
      f.lma.R = n;
      f.lma.threshold = -1.0f;
      f.lma.seed_out = e->d_seed;
      f.lma.seed_row = n - 1;
      f.lma.len_ptr = e->d_len;
      f.lma.len_advance = n;
    }
    if (engine_forward(e, f, s) != cudaSuccess) return DVLM_ERR_CUDA;
  }
  return DVLM_OK;
}

static dvlm_status check_cfg(dvlm_engine* e, const dvlm_decode_cfg* cfg) {
  if (!e || !cfg) return DVLM_ERR_INVALID_ARG;
  if (cfg->block_size < 1 || cfg->block_size > e->max_block) return DVLM_ERR_SHAPE;
  if (cfg->mode < DVLM_MODE_THRESHOLD || cfg->mode > DVLM_MODE_ROUTE) return DVLM_ERR_INVALID_ARG;
  if (cfg->mode == DVLM_MODE_SPEC_QUAD && !quad_supported(e, cfg->block_size)) return DVLM_ERR_UNSUPPORTED;
  if (cfg->mode == DVLM_MODE_ROUTE) {
    if (!e->bf16 || e->paged) return DVLM_ERR_UNSUPPORTED;
    if (cfg->route_k < 1 || cfg->route_n_vis < 0 || cfg->route_n_vis % 8 || cfg->block_size < 2) return DVLM_ERR_SHAPE;
  }
  if (std::isnan(cfg->threshold)) return DVLM_ERR_INVALID_ARG;
  if (cfg->ar_seed != 1) return DVLM_ERR_UNSUPPORTED;
  if (cfg->max_new_tokens < 1 || cfg->max_new_tokens > e->Lmax) return DVLM_ERR_SHAPE;
  return DVLM_OK;
}

dvlm_status dvlm_decode_block(dvlm_engine* e, const dvlm_decode_cfg* cfg, int32_t* out_tokens, int32_t* n_out,
                              dvlm_stats* stats, dvlm_stream stream) {
  const dvlm_status st = check_cfg(e, cfg);
  if (st != DVLM_OK) return st;
  if (!out_tokens || !n_out) return DVLM_ERR_INVALID_ARG;
  cudaStream_t s = cs(stream);
  int32_t L = 0;
  if (cudaMemcpyAsync(&L, e->d_len, 4, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return DVLM_ERR_CUDA;
  if (L + cfg->block_size > e->Lmax) return DVLM_ERR_CACHE_OVERFLOW;
  if (cudaMemsetAsync(e->n_out, 0, 4, s) != cudaSuccess) return DVLM_ERR_CUDA;
  int emitted = 0;
  const cudaError_t r = engine_step(e, *cfg, cfg->block_size, 0, &emitted, stats, s);
  if (r == cudaErrorLaunchTimeout) return DVLM_ERR_TIMEOUT;
  if (r != cudaSuccess) return DVLM_ERR_CUDA;
  if (emitted > 0 && cudaMemcpyAsync(out_tokens, e->stage_out, static_cast<size_t>(emitted) * 4,
                                     cudaMemcpyDeviceToDevice, s) != cudaSuccess)
    return DVLM_ERR_CUDA;
  if (stats) stats->n_tokens += emitted;
  if (engine_collect_stats(e, stats, s) != cudaSuccess) return DVLM_ERR_CUDA;
  *n_out = emitted;
  return DVLM_OK;
}

static dvlm_status generate_impl(dvlm_engine* e, const dvlm_decode_cfg* cfg, dvlm_stats* stats, cudaStream_t s) {
  e->quad_ready = false;  // a run starts from the pending seed: the quadratic mode drafts afresh
  int32_t L = 0;
  if (cudaMemcpyAsync(&L, e->d_len, 4, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return DVLM_ERR_CUDA;
  // worst case: every block/round ends B slots further (spec truncates back)
  if (static_cast<long long>(L) + cfg->max_new_tokens + cfg->block_size > e->Lmax) return DVLM_ERR_CACHE_OVERFLOW;
  if (cfg->mode == DVLM_MODE_ROUTE && cfg->route_n_vis > L) return DVLM_ERR_SHAPE;
  if (cudaMemsetAsync(e->n_out, 0, 4, s) != cudaSuccess) return DVLM_ERR_CUDA;
  int n = 0;
  while (n < cfg->max_new_tokens) {
    int emitted = 0;
    const cudaError_t r = engine_step(e, *cfg, cfg->max_new_tokens, n, &emitted, stats, s);
    if (r == cudaErrorLaunchTimeout) return DVLM_ERR_TIMEOUT;
    if (r != cudaSuccess) return DVLM_ERR_CUDA;
    n += emitted;
  }
  if (stats) stats->n_tokens += n;
  if (engine_collect_stats(e, stats, s) != cudaSuccess) return DVLM_ERR_CUDA;
  return DVLM_OK;
}

dvlm_status dvlm_generate(dvlm_engine* e, const dvlm_decode_cfg* cfg, int32_t* out_tokens, dvlm_stats* stats,
                          dvlm_stream stream) {
  const dvlm_status st = check_cfg(e, cfg);
  if (st != DVLM_OK) return st;
  if (!out_tokens) return DVLM_ERR_INVALID_ARG;
  cudaStream_t s = cs(stream);
  const dvlm_status g = generate_impl(e, cfg, stats, s);
  if (g != DVLM_OK) return g;
  return cuda_status(cudaMemcpyAsync(out_tokens, e->stage_out, static_cast<size_t>(cfg->max_new_tokens) * 4,
                                     cudaMemcpyDeviceToDevice, s));
}

dvlm_status dvlm_generate_host(dvlm_engine* e, const dvlm_decode_cfg* cfg, const void* vision_host, int n_vision,
                               const int32_t* ids_host, int n_ids, int32_t* out_host, dvlm_stats* stats,
                               dvlm_stream stream) {
  const dvlm_status st = check_cfg(e, cfg);
  if (st != DVLM_OK) return st;
  if (!out_host || (n_vision > 0 && !vision_host) || (n_ids > 0 && !ids_host)) return DVLM_ERR_INVALID_ARG;
  if (n_vision < 0 || n_ids < 0 || n_vision + n_ids > e->max_ctx) return DVLM_ERR_SHAPE;
  cudaStream_t s = cs(stream);
  const size_t es = e->bf16 ? 2 : 4;
  if (n_vision > 0 && cudaMemcpyAsync(e->stage_vis, vision_host, static_cast<size_t>(n_vision) * e->m.hidden * es,
                                      cudaMemcpyHostToDevice, s) != cudaSuccess)
    return DVLM_ERR_CUDA;
  if (n_ids > 0 &&
      cudaMemcpyAsync(e->stage_ids, ids_host, static_cast<size_t>(n_ids) * 4, cudaMemcpyHostToDevice, s) != cudaSuccess)
    return DVLM_ERR_CUDA;
  dvlm_status p = dvlm_prefill(e, n_vision > 0 ? e->stage_vis : nullptr, n_vision, n_ids > 0 ? e->stage_ids : nullptr,
                               n_ids, stream);
  if (p != DVLM_OK) return p;
  p = generate_impl(e, cfg, stats, s);
  if (p != DVLM_OK) return p;
  if (cudaMemcpyAsync(out_host, e->stage_out, static_cast<size_t>(cfg->max_new_tokens) * 4, cudaMemcpyDeviceToHost,
                      s) != cudaSuccess)
    return DVLM_ERR_CUDA;
  return cuda_status(cudaStreamSynchronize(s));
}

dvlm_status dvlm_engine_get_position(dvlm_engine* e, int32_t* L, int32_t* seed, dvlm_stream stream) {
  if (!e || !L || !seed) return DVLM_ERR_INVALID_ARG;
  cudaStream_t s = cs(stream);
  if (cudaMemcpyAsync(L, e->d_len, 4, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaMemcpyAsync(seed, e->d_seed, 4, cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return DVLM_ERR_CUDA;
  return cuda_status(cudaStreamSynchronize(s));
}

dvlm_status dvlm_engine_set_position(dvlm_engine* e, int32_t L, int32_t seed, dvlm_stream stream) {
  if (!e) return DVLM_ERR_INVALID_ARG;
  if (L < 0 || L > e->Lmax) return DVLM_ERR_SHAPE;
  if (seed < 0 || seed >= e->m.vocab) return DVLM_ERR_INVALID_ARG;
  e->quad_ready = false;
  cudaStream_t s = cs(stream);
  if (cudaMemcpyAsync(e->d_len, &L, 4, cudaMemcpyHostToDevice, s) != cudaSuccess ||
      cudaMemcpyAsync(e->d_seed, &seed, 4, cudaMemcpyHostToDevice, s) != cudaSuccess)
    return DVLM_ERR_CUDA;
  return cuda_status(cudaStreamSynchronize(s));
}

dvlm_status dvlm_engine_check(dvlm_engine* e, dvlm_stream stream) {
  if (!e) return DVLM_ERR_INVALID_ARG;
  cudaStream_t s = cs(stream);
  int h = 0;
  if (cudaStreamSynchronize(s) != cudaSuccess) return DVLM_ERR_CUDA;
  if (cudaMemcpy(&h, e->d_status, 4, cudaMemcpyDeviceToHost) != cudaSuccess) return DVLM_ERR_CUDA;
  if (cudaMemset(e->d_status, 0, 4) != cudaSuccess) return DVLM_ERR_CUDA;
  return static_cast<dvlm_status>(h);
}

dvlm_status dvlm_forward(dvlm_engine* e, const void* x_in, const int32_t* tokens, const uint8_t* masked, int n_rows,
                         int n_clean, int first_layer, int n_layers_run, int advance, void* x_out,
                         dvlm_stream stream) {
  if (!e) return DVLM_ERR_INVALID_ARG;
  if (n_rows < 1 || n_rows > kNT || n_clean < 0 || n_clean > n_rows) return DVLM_ERR_SHAPE;
  if (first_layer < 0 || n_layers_run < 0 || first_layer + n_layers_run > e->m.n_layers) return DVLM_ERR_SHAPE;
  if (!x_in && !tokens) return DVLM_ERR_INVALID_ARG;
  if (e->bf16 && x_in && !al16(x_in)) return DVLM_ERR_INVALID_ARG;
  cudaStream_t s = cs(stream);
  int32_t L = 0;
  if (cudaMemcpyAsync(&L, e->d_len, 4, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return DVLM_ERR_CUDA;
  if (L + n_rows > e->Lmax) return DVLM_ERR_CACHE_OVERFLOW;
  FwdSpec f;
  f.rows_in = x_in;
  f.n_src = x_in ? n_rows : 0;
  f.tokens = tokens;
  f.masked = masked;
  f.n_rows = n_rows;
  f.n_clean = n_clean;
  f.layer0 = first_layer;
  f.n_layers = n_layers_run;
  f.advance = advance != 0;
  f.x_out = x_out;
  return cuda_status(engine_forward(e, f, s));
}

dvlm_status dvlm_forward_text_only(dvlm_engine* e, const int32_t* tokens, const uint8_t* masked, int n_rows,
                                   int n_hidden, void* x_out, dvlm_stream stream) {
  if (!e || !tokens) return DVLM_ERR_INVALID_ARG;
  if (!e->bf16 || e->paged) return DVLM_ERR_UNSUPPORTED;
  if (n_rows < 1 || n_rows > kNT || n_hidden < 0 || n_hidden % 8) return DVLM_ERR_SHAPE;
  if (x_out && !al16(x_out)) return DVLM_ERR_INVALID_ARG;
  cudaStream_t s = cs(stream);
  int32_t L = 0;
  if (cudaMemcpyAsync(&L, e->d_len, 4, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return DVLM_ERR_CUDA;
  if (L + n_rows > e->Lmax) return DVLM_ERR_CACHE_OVERFLOW;
  if (n_hidden > L) return DVLM_ERR_SHAPE;
  FwdSpec f;
  f.tokens = tokens;
  f.masked = masked;
  f.n_rows = n_rows;
  f.n_clean = 0;
  f.x_out = x_out;
  f.hide = n_hidden;
  f.L_host = L;
  return cuda_status(engine_forward(e, f, s));
}

dvlm_status dvlm_profile_forward(dvlm_engine* e, const int32_t* tokens, const uint8_t* masked, int n_rows,
                                 int n_clean, int with_lm_head, float* ms_out, int* counts_out, dvlm_stream stream) {
  if (!e || !tokens || !ms_out || !counts_out) return DVLM_ERR_INVALID_ARG;
  if (n_rows < 1 || n_rows > kNT || n_clean < 0 || n_clean > n_rows) return DVLM_ERR_SHAPE;
  if (!e->bf16) return DVLM_ERR_UNSUPPORTED;
  cudaStream_t s = cs(stream);
  int32_t L = 0;
  if (cudaMemcpyAsync(&L, e->d_len, 4, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return DVLM_ERR_CUDA;
  if (L + n_rows > e->Lmax) return DVLM_ERR_CACHE_OVERFLOW;
  FwdSpec f;
  f.tokens = tokens;
  f.masked = masked;
  f.n_rows = n_rows;
  f.n_clean = n_clean;
  f.lm = with_lm_head != 0;
  f.lma.R = n_rows;
  f.lma.threshold = -1.0f;
  return cuda_status(engine_profile(e, f, ms_out, counts_out, s));
}

dvlm_status dvlm_selftest_wait_timeout(long long budget_cycles, int* dev_status, int* gave_up,
                                       dvlm_stream stream) {
  if (!dev_status || !gave_up) return DVLM_ERR_INVALID_ARG;
  if (budget_cycles < 1 || budget_cycles > 4000000000LL) return DVLM_ERR_SHAPE;
  return cuda_status(launch_selftest_timeout(budget_cycles, dev_status, gave_up, cs(stream)));
}

dvlm_status dvlm_engine_set_option(dvlm_engine* e, const char* name, int value) {
  if (!e || !name) return DVLM_ERR_INVALID_ARG;
  if (!e->bf16) return DVLM_ERR_UNSUPPORTED;
  return engine_set_option(e, name, value);
}

dvlm_status dvlm_engine_set_paged(dvlm_engine* e, void* k_pages, void* v_pages, const int32_t* block_table,
                                  int n_pages, int max_pages) {
  if (!e || !k_pages || !v_pages || !block_table) return DVLM_ERR_INVALID_ARG;
  if (!e->bf16) return DVLM_ERR_UNSUPPORTED;
  if (n_pages < 1 || max_pages < 1 || static_cast<long long>(max_pages) * 64 < e->Lmax) return DVLM_ERR_SHAPE;
  if (!al16(k_pages) || !al16(v_pages)) return DVLM_ERR_INVALID_ARG;
  return engine_set_paged(e, k_pages, v_pages, block_table, n_pages, max_pages) ? DVLM_OK : DVLM_ERR_CUDA;
}

dvlm_status dvlm_forward_quad(dvlm_engine* e, const int32_t* draft, int B, void* x_out, dvlm_stream stream) {
  if (!e || !draft || !x_out) return DVLM_ERR_INVALID_ARG;
  if (B < 1 || B > kNT || B + B * B > e->max_ctx) return DVLM_ERR_SHAPE;
  if (!quad_supported(e, B)) return DVLM_ERR_UNSUPPORTED;
  if (!al16(x_out)) return DVLM_ERR_INVALID_ARG;
  cudaStream_t s = cs(stream);
  int32_t L = 0;
  if (cudaMemcpyAsync(&L, e->d_len, 4, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return DVLM_ERR_CUDA;
  if (L + 2 * B > e->Lmax) return DVLM_ERR_CACHE_OVERFLOW;
  e->quad_ready = false;
  return cuda_status(engine_forward_quad(e, draft, B, x_out, s));
}

size_t dvlm_engine_trace_record_bytes(const dvlm_model* m) {
  if (!model_ok(m)) return 0;
  return trace_record_bytes(m->hidden, m->dtype != DVLM_FP32);
}

dvlm_status dvlm_engine_set_trace(dvlm_engine* e, void* buf, size_t bytes, int32_t* count) {
  if (!e) return DVLM_ERR_INVALID_ARG;
  if (!buf) {
    engine_set_trace(e, nullptr, 0, nullptr);
    return DVLM_OK;
  }
  if (!count || !al16(buf) || !al16(count)) return DVLM_ERR_INVALID_ARG;
  const size_t rb = trace_record_bytes(e->m.hidden, e->bf16);
  if (bytes < rb) return DVLM_ERR_WORKSPACE;
  const size_t cap = bytes / rb;
  engine_set_trace(e, buf, static_cast<int>(cap > 1000000 ? 1000000 : cap), count);
  return DVLM_OK;
}

int dvlm_engine_get_option(dvlm_engine* e, const char* name) {
  if (!e || !name) return -1;
  return engine_get_option(e, name);
}

}  // extern "C"
