// Decode engine: forward orchestration (PDL-chained kernels, CUDA graphs),
// prefill and the three decoding drivers.
//
//   threshold [Fast-dVLM technical overview (ocdem.com), sections 2.2.1,
//     2.2.2, 4.1]: per block, position 0 is the AR seed; noisy passes over
//     the whole block score the still-masked positions (position j from row
//     j-1) and commit those with top-1 probability >= threshold (at least
//     one); a causal pass over the finished block then makes its K/V final,
//     advances L by B and seeds the next block from its last row;
//   linear self-speculative [same page, section 2.3.1]: one noisy draft pass
//     commits every position, one causal verify pass scores the draft, the
//     longest agreeing prefix is kept and L is truncated to it;
//   AR: one causal row per pass (the comparator).
#include <cmath>
#include <cstring>
#include <string>

#include "engine.h"
#include "ptx.cuh"

using namespace dvlm;

namespace dvlm {

cudaError_t launch_topk_commit(const float* p1, const int32_t* ids, const int32_t* other_ids, uint8_t* masked,
                               int32_t* tokens, int R, int k, uint8_t* commit, int32_t* n_commit, cudaStream_t s);

__global__ void advance_kernel(int32_t* d_len, int n) {
  griddep_wait();
  griddep_launch_dependents();
  if (threadIdx.x == 0) *d_len += n;
}

static size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Forward trace (test hook): the block state before a forward ...
__global__ void trace_begin_kernel(uint8_t* buf, size_t rec_bytes, int cap, const int32_t* cnt, int kind,
                                   const int32_t* d_len, int n_rows, int n_clean, int R, const int32_t* tokens,
                                   const uint8_t* masked) {
  const int idx = *cnt;
  if (idx >= cap) return;
  int32_t* w = reinterpret_cast<int32_t*>(buf + static_cast<size_t>(idx) * rec_bytes);
  const int t = threadIdx.x;
  if (t < 8) w[t] = t == 0 ? kind : t == 1 ? *d_len : t == 2 ? n_rows : t == 3 ? n_clean : t == 4 ? R : 0;
  if (t < kNT) {
    w[8 + t] = t < n_rows ? tokens[t] : -1;
    w[24 + t] = (t < n_rows && masked) ? static_cast<int32_t>(masked[t]) : 0;
  }
}

// ... and after it: LM-head outputs, the block state, the next seed and cache
// length, and the final residual stream rows; then the record count advances.
__global__ void trace_end_kernel(uint8_t* buf, size_t rec_bytes, int cap, int32_t* cnt, const int32_t* d_len,
                                 const int32_t* d_seed, int n_rows, int R, const int32_t* top1, const float* p1,
                                 const int32_t* tokens, const uint8_t* masked, const uint8_t* x, size_t x_bytes) {
  const int idx = *cnt;
  if (idx < cap) {
    uint8_t* rec = buf + static_cast<size_t>(idx) * rec_bytes;
    int32_t* w = reinterpret_cast<int32_t*>(rec);
    const int t = threadIdx.x;
    if (t < kNT) {
      w[40 + t] = t < R ? top1[t] : -1;
      w[56 + t] = t < R ? __float_as_int(p1[t]) : 0;
      w[72 + t] = t < n_rows ? tokens[t] : -1;
      w[88 + t] = (t < n_rows && masked) ? static_cast<int32_t>(masked[t]) : 0;
    }
    if (t < 8) w[104 + t] = t == 0 ? *d_seed : t == 1 ? *d_len : 0;
    uint8_t* xr = rec + kTraceWords * 4;
    for (size_t i = t; i < x_bytes / 4; i += blockDim.x)
      reinterpret_cast<uint32_t*>(xr)[i] = reinterpret_cast<const uint32_t*>(x)[i];
  }
  __syncthreads();
  if (threadIdx.x == 0 && idx < cap) *cnt = idx + 1;
}

struct Carver {
  uint8_t* base;
  size_t off = 0;
  bool dry;
  template <class T>
  T* take(size_t bytes) {
    off = align_up(off, 256);
    T* p = dry ? nullptr : reinterpret_cast<T*>(base + off);
    off += bytes;
    return p;
  }
};

static int num_tiles_max(const dvlm_model& m) {
  const int qkv_rows = (m.n_q_heads + 2 * m.n_kv_heads) * m.head_dim;
  int t = std::max(qkv_rows / 128, m.hidden / 128);
  t = std::max(t, m.inter / 64);
  t = std::max(t, (m.vocab + 127) / 128);
  return t;
}

// Lays the workspace out (or measures it when dry).
static size_t carve(dvlm_engine* e, uint8_t* base, bool dry, int P) {
  const dvlm_model& m = e->m;
  const size_t es = e->bf16 ? 2 : 4;
  const int H = m.hidden, I = m.inter, HD = m.n_q_heads * m.head_dim;
  const int qkv_rows = (m.n_q_heads + 2 * m.n_kv_heads) * m.head_dim;
  Carver c{base, 0, dry};
  e->x = c.take<void>(kNT * H * es);
  e->q = c.take<void>(kNT * HD * es);
  e->attn_o = c.take<void>(kNT * HD * es);
  e->act = c.take<void>(static_cast<size_t>(kNT) * I * es);
  // sums of squares per (128-feature tile, cluster CTA): up to 16 CTAs per tile
  e->ssq = c.take<float>(((H / 128) * 16 + 1) * kNT * 4);
  e->gpart = c.take<float>(gemm_ws_part_bytes(kNT, 2 * P));  // up to two CTAs per SM
  e->gcnt_stride = num_tiles_max(m);
  e->gcnt = c.take<int>(static_cast<size_t>(e->gcnt_stride) * 4 * 4);  // one block per GEMM kind of the persistent forward
  e->chain_bar = c.take<int>(2 * 4);
  e->lpart = c.take<float>(static_cast<size_t>(P) * kNT * 128 * 4);
  e->lcnt = c.take<int>(((m.vocab + 127) / 128) * 4);
  e->lrec = c.take<float>(static_cast<size_t>(P) * kNT * 16);
  e->ldone = c.take<int>(4);
  e->d_len = c.take<int32_t>(4);
  e->d_seed = c.take<int32_t>(4);
  e->d_status = c.take<int>(4);
  e->n_remaining = c.take<int32_t>(4);
  e->n_out = c.take<int32_t>(4);
  e->tokens = c.take<int32_t>((kNT + 1) * 4);
  e->vids = c.take<int32_t>((kNT + 1) * 4);
  e->masked = c.take<uint8_t>(kNT + 1);
  e->tr_top1 = c.take<int32_t>(kNT * 4);
  e->tr_p1 = c.take<float>(kNT * 4);
  e->anc_id = c.take<int32_t>(kNT * 4);
  e->anc_p1 = c.take<float>(kNT * 4);
  e->txt_id = c.take<int32_t>(kNT * 4);
  e->txt_p1 = c.take<float>(kNT * 4);
  e->cert = c.take<int32_t>(4);
  e->hist = c.take<int64_t>(DVLM_HIST * 8);
  e->ahist = c.take<int64_t>(DVLM_HIST * 8);
  e->stage_vis = c.take<void>(static_cast<size_t>(std::max(e->max_ctx, 1)) * H * es);
  e->stage_ids = c.take<int32_t>(std::max(e->max_ctx, 1) * 4);
  e->stage_out = c.take<int32_t>(static_cast<size_t>(e->Lmax) * 4);
  if (e->fp8) e->amax_act = c.take<float>(static_cast<size_t>(I / 64) * kNT * 4);
  if (e->bf16) e->attn_scratch = c.take<void>(attn_split_scratch_bytes(m.n_kv_heads, kMaxAttnSplit));
  if (e->bf16 && !e->fp8) e->fwd_att = c.take<void>(fwd_attn_scratch_bytes(m.n_kv_heads, e->Lmax));
  if (e->bf16 && !e->fp8 && e->max_ctx > 0) {
    const size_t C = static_cast<size_t>(e->max_ctx);
    e->px = c.take<void>(C * H * 2);
    e->pq = c.take<void>(C * HD * 2);
    e->pao = c.take<void>(C * HD * 2);
    e->pact = c.take<void>(C * I * 2);
    e->pssq = c.take<float>(static_cast<size_t>(std::max(H / 128 + 1, (H / 256) * 16)) * C * 4);
    e->rope_cs = c.take<float2>(C * 64 * 8);
    e->qtok = c.take<int32_t>(C * 4);
    e->d_k = c.take<int32_t>(4);
    e->kside = c.take<void>(static_cast<size_t>(m.n_kv_heads) * kQuadSideKeys * 128 * 2);
    e->vside = c.take<void>(static_cast<size_t>(m.n_kv_heads) * kQuadSideKeys * 128 * 2);
    e->qpart = c.take<float>(static_cast<size_t>(P) * 128 * 256 * 4);
    e->qcnt = c.take<int>(1024 * 4);
  }
  if (!e->bf16) {
    e->f_y = c.take<float>(static_cast<size_t>(kNT) * std::max(qkv_rows, H) * 4);
    e->f_r = c.take<float>(kNT * 4);
    e->f_g = c.take<float>(static_cast<size_t>(kNT) * I * 4);
    e->f_u = c.take<float>(static_cast<size_t>(kNT) * I * 4);
    e->f_p1 = c.take<float>(kNT * 4);
    e->f_id = c.take<int32_t>(kNT * 4);
  }
  return align_up(c.off, 256);
}

static bool build_maps(dvlm_engine* e) {
  const dvlm_model& m = e->m;
  const int H = m.hidden, I = m.inter, D = m.head_dim, Hq = m.n_q_heads, Hkv = m.n_kv_heads, L = m.n_layers;
  const int qkv_rows = (Hq + 2 * Hkv) * D;
  bool ok = true;
  if (e->fp8) {  // E4M3 codes: 128-byte (128 k) boxes
    ok &= make_tmap_2d_u8(&e->tm_wqkv, m.wqkv, H, static_cast<uint64_t>(L) * qkv_rows, H, 128, 128);
    ok &= make_tmap_2d_u8(&e->tm_wo, m.wo, Hq * D, static_cast<uint64_t>(L) * H, Hq * D, 128, 128);
    ok &= make_tmap_2d_u8(&e->tm_wg, m.wgate, H, static_cast<uint64_t>(L) * I, H, 128, 64);
    ok &= make_tmap_2d_u8(&e->tm_wu, m.wup, H, static_cast<uint64_t>(L) * I, H, 128, 64);
    ok &= make_tmap_2d_u8(&e->tm_wd, m.wdown, I, static_cast<uint64_t>(L) * H, I, 128, 128);
  } else {
    ok &= make_tmap_2d(&e->tm_wqkv, m.wqkv, H, static_cast<uint64_t>(L) * qkv_rows, H * 2, 64, 128);
    ok &= make_tmap_2d(&e->tm_wo, m.wo, Hq * D, static_cast<uint64_t>(L) * H, Hq * D * 2, 64, 128);
    ok &= make_tmap_2d(&e->tm_wg, m.wgate, H, static_cast<uint64_t>(L) * I, H * 2, 64, 64);
    ok &= make_tmap_2d(&e->tm_wu, m.wup, H, static_cast<uint64_t>(L) * I, H * 2, 64, 64);
    ok &= make_tmap_2d(&e->tm_wd, m.wdown, I, static_cast<uint64_t>(L) * H, static_cast<uint64_t>(I) * 2, 64, 128);
  }
  ok &= make_tmap_2d(&e->tm_lm, m.lm_head, H, m.vocab, H * 2, 64, 128);
  ok &= make_tmap_2d(&e->tm_x, e->x, H, kNT, H * 2, 64, kNT);
  ok &= make_tmap_2d(&e->tm_ao, e->attn_o, Hq * D, kNT, Hq * D * 2, 64, kNT);
  ok &= make_tmap_2d(&e->tm_act, e->act, I, kNT, static_cast<uint64_t>(I) * 2, 64, kNT);
  ok &= make_tmap_3d(&e->tm_q, e->q, D, Hq, kNT, D * 2, static_cast<uint64_t>(Hq) * D * 2, 64, 8, 16);
  ok &= make_tmap_2d(&e->tm_k, e->kc, D, static_cast<uint64_t>(L) * Hkv * e->Lmax, D * 2, 64, 64);
  ok &= make_tmap_2d(&e->tm_v, e->vc, e->Lmax, static_cast<uint64_t>(L) * Hkv * D,
                     static_cast<uint64_t>(e->Lmax) * 2, 64, 128);
  if (e->max_ctx > 0 && !e->fp8) {
    const uint64_t C = static_cast<uint64_t>(e->max_ctx);
    ok &= make_tmap_2d(&e->tm_px, e->px, H, C, H * 2, 64, 128);
    ok &= make_tmap_2d(&e->tm_pq, e->pq, Hq * D, C, Hq * D * 2, 64, 128);
    ok &= make_tmap_2d(&e->tm_pao, e->pao, Hq * D, C, Hq * D * 2, 64, 128);
    ok &= make_tmap_2d(&e->tm_pact, e->pact, I, C, static_cast<uint64_t>(I) * 2, 64, 128);
    ok &= make_tmap_2d(&e->tm_wqkv_p, m.wqkv, H, static_cast<uint64_t>(L) * qkv_rows, H * 2, 64, 256);
    ok &= make_tmap_2d(&e->tm_wo_p, m.wo, Hq * D, static_cast<uint64_t>(L) * H, Hq * D * 2, 64, 256);
    ok &= make_tmap_2d(&e->tm_wd_p, m.wdown, I, static_cast<uint64_t>(L) * H, static_cast<uint64_t>(I) * 2, 64, 256);
    ok &= make_tmap_2d(&e->tm_wg_p, m.wgate, H, static_cast<uint64_t>(L) * I, H * 2, 64, 128);
    ok &= make_tmap_2d(&e->tm_wu_p, m.wup, H, static_cast<uint64_t>(L) * I, H * 2, 64, 128);
    ok &= make_tmap_2d(&e->tm_kp, e->kc, D, static_cast<uint64_t>(L) * Hkv * e->Lmax, D * 2, 64, 128);
    ok &= make_tmap_3d(&e->tm_q3, e->pq, D, Hq, C, D * 2, static_cast<uint64_t>(Hq) * D * 2, 64, 8, 16);
    ok &= make_tmap_2d(&e->tm_ks, e->kside, D, static_cast<uint64_t>(Hkv) * kQuadSideKeys, D * 2, 64, 64);
    ok &= make_tmap_2d(&e->tm_vs, e->vside, kQuadSideKeys, static_cast<uint64_t>(Hkv) * D, kQuadSideKeys * 2, 64,
                       128);
  }
  return ok;
}



static int ws_ctas(dvlm_engine* e, long long units) {
  return static_cast<int>(std::min<long long>(e->sm, units));
}

static void fill_lm_scratch(dvlm_engine* e, LmArgs& a) {
  a.part = e->lpart;
  a.cnt = e->lcnt;
  a.rec = e->lrec;
  a.done = e->ldone;
  a.status = e->d_status;
  a.V = e->m.vocab;
}

#define DVLM_CK(x)                            \
  do {                                        \
    cudaError_t err__ = (x);                  \
    if (err__ != cudaSuccess) return err__;   \
  } while (0)

// Persistent forward (one launch for all layers): bf16 weights, 128-wide
// heads, 8 query heads per KV head, feature counts in whole tiles, and one
// resident CTA on every SM.
static bool persistent_supported(dvlm_engine* e) {
  const dvlm_model& m = e->m;
  return e->bf16 && !e->fp8 && m.head_dim == 128 && m.hidden % 128 == 0 && m.inter % 64 == 0 &&
         m.n_q_heads == 8 * m.n_kv_heads && e->Lmax <= 8192 && e->fwd_att && e->sm >= 1 &&
         e->sm <= fwd_persistent_max_ctas();
}

static ChainPhase chain_phase(const CUtensorMap& a, const CUtensorMap& a2, const CUtensorMap& b, int n_tiles, int kb,
                              const GemmEpi& ea, int* cnt) {
  ChainPhase ph{};
  ph.mapA = a;
  ph.mapA2 = a2;
  ph.mapB = b;
  ph.ea = ea;
  ph.ea.cnt = cnt;
  ph.n_tiles = n_tiles;
  ph.kb = kb;
  return ph;
}

static cudaError_t fwd_bf16(dvlm_engine* e, const FwdSpec& f, cudaStream_t s) {
  const dvlm_model& m = e->m;
  const int H = m.hidden, I = m.inter, D = m.head_dim, Hq = m.n_q_heads, Hkv = m.n_kv_heads;
  const int qkv_rows = (Hq + 2 * Hkv) * D;
  const bool pdl = e->pdl;
  bf16* x = static_cast<bf16*>(e->x);
  KernelTimer* tm = f.timer;
  auto T0 = [&](int k) { if (tm) tm->begin(k); };
  auto T1 = [&](int k) { if (tm) tm->end(k); };
  // TEXT-ONLY pass [Look Only When Needed, method step (2): the vision rows
  // removed, position ids kept]: attention reads the cache from slot f.hide
  // on.  The K and V^T maps start f.hide slots in and end where the cache
  // allocation ends (outer rows of K, inner keys of V^T shortened by f.hide),
  // so a 64-key box past the last valid key is zero-filled instead of read
  // beyond the allocation; the length is the host-read L minus f.hide.  The
  // QKV epilogue still writes K/V at the absolute slots.
  CUtensorMap tm_k_text, tm_v_text;
  if (f.hide > 0) {
    const uint64_t k_rows = static_cast<uint64_t>(m.n_layers) * Hkv * e->Lmax;
    bool ok = make_tmap_2d(&tm_k_text, static_cast<const bf16*>(e->kc) + static_cast<size_t>(f.hide) * D, D,
                           k_rows - f.hide, D * 2, 64, 64);
    ok &= make_tmap_2d(&tm_v_text, static_cast<const bf16*>(e->vc) + f.hide, e->Lmax - f.hide,
                       static_cast<uint64_t>(m.n_layers) * Hkv * D, static_cast<uint64_t>(e->Lmax) * 2, 64, 128);
    if (!ok) return cudaErrorInvalidValue;
  }
  T0(K_EMBED);
  DVLM_CK(launch_embed_bf16(static_cast<const bf16*>(m.embed), static_cast<const bf16*>(f.rows_in), f.n_src,
                            f.tokens, f.masked, m.mask_id, f.n_rows, H, m.vocab, x, e->ssq, kNT, e->d_status, pdl,
                            s));
  T1(K_EMBED);
  const int l1 = f.n_layers < 0 ? m.n_layers : f.layer0 + f.n_layers;
  GemmEpi ea{};
  ea.n_rows = f.n_rows;
  ea.ssq_in = e->ssq;
  // entries of the sums-of-squares buffer the next RMSNorm adds up: one per
  // 128-feature tile from the embedding and stream-K projections, one per
  // (tile, cluster CTA) from the cluster split-K projections
  int n_ssq = H / 128;
  ea.inv_h = 1.0f / H;
  ea.eps = m.eps;
  ea.Lmax = e->Lmax;
  ea.n_q_heads = Hq;
  ea.n_kv_heads = Hkv;
  ea.d_len = e->d_len;
  ea.log2_rope_base = std::log2(static_cast<double>(m.rope_base));
  ea.part = e->gpart;
  ea.cnt = e->gcnt;
  ea.status = e->d_status;
  // per-layer cache stride: contiguous [Hkv][Lmax][D], or paged [n_pages][Hkv][64][D]
  const size_t kv_layer = e->paged ? static_cast<size_t>(e->n_pages) * Hkv * 64 * D
                                   : static_cast<size_t>(Hkv) * e->Lmax * D;
  if (e->paged) {
    ea.block_table = e->block_table;
    ea.n_pages = e->n_pages;
  }
  // the whole forward as one persistent launch (contiguous cache, no hidden
  // slots): first layer's QKV, then per layer attention, merge, O, gate/up,
  // down and the next layer's QKV
  const bool persistent = e->chain && !e->fp8 && !e->paged && f.hide == 0;
  if (persistent) {
    const GemmEpi base = ea;
    FwdProgram fp{};
    GemmEpi q = base;
    q.epi = EPI_QKV;
    q.n_ssq = H / 128;
    q.out = static_cast<bf16*>(e->q);
    q.out_ld = Hq * D;
    q.kcache = static_cast<bf16*>(e->kc);
    q.vcache = static_cast<bf16*>(e->vc);
    GemmEpi o = base;  // O-projection and down: residual add + sums of squares
    o.epi = EPI_RESID;
    o.resid = x;
    o.resid_ld = H;
    o.ssq_out = e->ssq;
    GemmEpi g = base;
    g.epi = EPI_SWIGLU;
    g.n_ssq = H / 128;
    g.out = static_cast<bf16*>(e->act);
    g.out_ld = I;
    const int cs = e->gcnt_stride;
    fp.qkv = chain_phase(e->tm_wqkv, e->tm_wqkv, e->tm_x, qkv_rows / 128, H / 64, q, e->gcnt);
    fp.o = chain_phase(e->tm_wo, e->tm_wo, e->tm_ao, H / 128, Hq * D / 64, o, e->gcnt + cs);
    fp.gu = chain_phase(e->tm_wg, e->tm_wu, e->tm_x, I / 64, H / 64, g, e->gcnt + 2 * cs);
    fp.down = chain_phase(e->tm_wd, e->tm_wd, e->tm_act, H / 128, I / 64, o, e->gcnt + 3 * cs);
    // the narrow QKV and O products one tile per CTA (no split tiles to add
    // up across CTAs; their weights are prefetched during the phases before)
    fp.qkv.ctas = qkv_rows / 128;
    fp.o.ctas = H / 128;
    fp.qkv_rows = qkv_rows;
    fp.H = H;
    fp.I = I;
    fp.kv_layer = kv_layer;
    fp.mapQ = e->tm_q;
    fp.mapK = e->tm_k;
    fp.mapV = e->tm_v;
    fp.Hq = Hq;
    fp.Hkv = Hkv;
    fp.Lmax = e->Lmax;
    fp.n_clean = f.n_clean;
    fp.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(D)));
    fp.apart = static_cast<float*>(e->fwd_att);
    fp.n_chunks_max = (e->Lmax + 63) / 64;
    fp.aml = reinterpret_cast<float2*>(static_cast<uint8_t*>(e->fwd_att) +
                                       (static_cast<size_t>(Hkv) * fp.n_chunks_max * 128 * 128 * 4 + 255) / 256 * 256);
    fp.attn_o = static_cast<bf16*>(e->attn_o);
    fp.layer0 = f.layer0;
    fp.n_layers = l1 - f.layer0;
    fp.bar = e->chain_bar;
    fp.status = e->d_status;
    T0(K_CHAIN);
    DVLM_CK(launch_fwd_persistent(fp, e->sm, pdl, s));
    T1(K_CHAIN);
    n_ssq = H / 128;
  }
  for (int l = f.layer0; l < l1 && !persistent; ++l) {
    ea.epi = EPI_QKV;
    ea.n_ssq = n_ssq;
    ea.out = static_cast<bf16*>(e->q);
    ea.out_ld = Hq * D;
    ea.kcache = static_cast<bf16*>(e->kc) + l * kv_layer;
    ea.vcache = static_cast<bf16*>(e->vc) + l * kv_layer;
    T0(K_QKV);
    if (e->fp8) {  // W8A8 [Fast-dVLM technical overview (ocdem.com), section 2.3.2]
      ea.q_src = x;
      ea.q_ld = H;
      ea.q_K = H;
      ea.rms_input = 1;
      ea.amax_in = nullptr;
      ea.wscale = m.sqkv;
      if (e->s_qkv > 0)
        DVLM_CK(launch_gemm_cl_fp8(e->tm_wqkv, qkv_rows / 128, H / 128, e->s_qkv, l * qkv_rows, ea, pdl, s, 5));
      else
        DVLM_CK(launch_gemm_ws_fp8(e->tm_wqkv, e->tm_wqkv, qkv_rows / 128, H / 128,
                                   ws_ctas(e, (qkv_rows / 128) * (H / 128)), l * qkv_rows, ea, pdl, s));
    } else if (e->s_qkv > 0) {
      DVLM_CK(launch_gemm_cl(kNT, e->tm_wqkv, e->tm_x, qkv_rows / 128, H / 64, e->s_qkv, l * qkv_rows, ea, pdl, s,
                             5));
    } else {
      DVLM_CK(launch_gemm_ws(kNT, e->tm_wqkv, e->tm_wqkv, e->tm_x, qkv_rows / 128, H / 64,
                             ws_ctas(e, (qkv_rows / 128) * (H / 64)), l * qkv_rows, ea, pdl, s, 5));
    }
    T1(K_QKV);
    AttnArgs aa{};
    aa.n_rows = f.n_rows;
    aa.n_clean = f.n_clean;
    aa.n_batch = 1;
    aa.d_len = e->d_len;
    aa.Lmax = e->Lmax;
    aa.Hq = Hq;
    aa.Hkv = Hkv;
    aa.kv_base = l;
    aa.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(D)));
    aa.out = static_cast<bf16*>(e->attn_o);
    aa.status = e->d_status;
    if (e->paged) {
      aa.block_table = e->block_table;
      aa.max_pages = e->max_pages;
      aa.n_pages = e->n_pages;
    }
    T0(K_ATTN);
    if (f.hide > 0) aa.len_sub = f.hide;  // the view starts f.hide slots into the cache
    const CUtensorMap& mk = f.hide > 0 ? tm_k_text : e->tm_k;
    const CUtensorMap& mv = f.hide > 0 ? tm_v_text : e->tm_v;
    if (e->attn_split > 0)
      DVLM_CK(launch_attn_split(e->tm_q, mk, mv, aa, e->attn_split, e->attn_scratch, pdl, s));
    else
      DVLM_CK(launch_attn_split_cl(e->tm_q, mk, mv, aa, e->attn_cs, pdl, s));
    T1(K_ATTN);
    ea.epi = EPI_RESID;
    ea.resid = x;
    ea.resid_ld = H;
    ea.ssq_out = e->ssq;
    T0(K_OPROJ);
    if (e->fp8) {
      ea.q_src = static_cast<bf16*>(e->attn_o);
      ea.q_ld = Hq * D;
      ea.q_K = Hq * D;
      ea.rms_input = 0;
      ea.amax_in = nullptr;
      ea.wscale = m.so;
      if (e->s_o > 0)
        DVLM_CK(launch_gemm_cl_fp8(e->tm_wo, H / 128, Hq * D / 128, e->s_o, l * H, ea, pdl, s, 5));
      else
        DVLM_CK(launch_gemm_ws_fp8(e->tm_wo, e->tm_wo, H / 128, Hq * D / 128, ws_ctas(e, (H / 128) * (Hq * D / 128)),
                                   l * H, ea, pdl, s));
    } else if (e->s_o > 0) {
      DVLM_CK(launch_gemm_cl(kNT, e->tm_wo, e->tm_ao, H / 128, Hq * D / 64, e->s_o, l * H, ea, pdl, s, 5));
    } else {
      DVLM_CK(launch_gemm_ws(kNT, e->tm_wo, e->tm_wo, e->tm_ao, H / 128, Hq * D / 64,
                             ws_ctas(e, (H / 128) * (Hq * D / 64)), l * H, ea, pdl, s, 5));
    }
    T1(K_OPROJ);
    n_ssq = (H / 128) * (e->s_o > 0 ? e->s_o : 1);
    ea.epi = EPI_SWIGLU;
    ea.n_ssq = n_ssq;
    ea.out = static_cast<bf16*>(e->act);
    ea.out_ld = I;
    T0(K_GATEUP);
    if (e->fp8) {
      ea.q_src = x;
      ea.q_ld = H;
      ea.q_K = H;
      ea.rms_input = 1;
      ea.amax_in = nullptr;
      ea.wscale = m.sgate;
      ea.wscale2 = m.sup;
      ea.amax_out = e->amax_act;
      const long long units = static_cast<long long>(I / 64) * (H / 128);
      DVLM_CK(launch_gemm_ws_fp8(e->tm_wg, e->tm_wu, I / 64, H / 128,
                                 static_cast<int>(std::min<long long>(units, e->sm)), l * I, ea, pdl, s));
    } else {
      const long long gu_units = static_cast<long long>(I / 64) * (H / 64);
      const int gu_ctas = static_cast<int>(std::min<long long>(gu_units, static_cast<long long>(e->gu_cps) * e->sm));
      DVLM_CK(launch_gemm_ws(kNT, e->tm_wg, e->tm_wu, e->tm_x, I / 64, H / 64, gu_ctas,
                             l * I, ea, pdl, s, e->gu_stages));
    }
    T1(K_GATEUP);
    ea.epi = EPI_RESID;
    T0(K_DOWN);
    if (e->fp8) {
      ea.q_src = static_cast<bf16*>(e->act);
      ea.q_ld = I;
      ea.q_K = I;
      ea.rms_input = 0;
      ea.amax_in = e->amax_act;
      ea.n_amax = I / 64;
      ea.wscale = m.sdown;
      ea.wscale2 = nullptr;
      ea.amax_out = nullptr;
      if (e->s_down <= 0) return cudaErrorInvalidValue;  // the fp8 down projection runs split-K in clusters
      DVLM_CK(launch_gemm_cl_fp8(e->tm_wd, H / 128, I / 128, e->s_down, l * H, ea, pdl, s, e->down_stages));
    } else if (e->s_down > 0) {
      DVLM_CK(launch_gemm_cl(kNT, e->tm_wd, e->tm_act, H / 128, I / 64, e->s_down, l * H, ea, pdl, s,
                             e->down_stages));
    } else {
      DVLM_CK(launch_gemm_ws(kNT, e->tm_wd, e->tm_wd, e->tm_act, H / 128, I / 64,
                             ws_ctas(e, (H / 128) * (I / 64)), l * H, ea, pdl, s, e->down_stages));
    }
    T1(K_DOWN);
    n_ssq = (H / 128) * (e->s_down > 0 ? e->s_down : 1);
  }
  if (f.x_out) DVLM_CK(cudaMemcpyAsync(f.x_out, x, static_cast<size_t>(f.n_rows) * H * 2, cudaMemcpyDeviceToDevice, s));
  if (f.lm) {
    LmArgs a = f.lma;
    fill_lm_scratch(e, a);
    a.ssq_in = e->ssq;
    a.n_ssq = n_ssq;
    a.inv_h = 1.0f / H;
    a.eps = m.eps;
    const int nt = (m.vocab + 127) / 128;
    T0(K_LMHEAD);
    DVLM_CK(launch_lmhead(kNT, e->tm_lm, e->tm_x, nt, H / 64, ws_ctas(e, static_cast<long long>(nt) * (H / 64)), a,
                          pdl, s));
    T1(K_LMHEAD);
  } else if (f.advance) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(1);
    cfg.blockDim = dim3(32);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    DVLM_CK(cudaLaunchKernelEx(&cfg, advance_kernel, e->d_len, f.n_rows));
  }
  return cudaSuccess;
}

static cudaError_t fwd_f32(dvlm_engine* e, const FwdSpec& f, cudaStream_t s) {
  const dvlm_model& m = e->m;
  const int H = m.hidden, I = m.inter, D = m.head_dim, Hq = m.n_q_heads, Hkv = m.n_kv_heads;
  const int qkv_rows = (Hq + 2 * Hkv) * D;
  const int n = f.n_rows;
  float* x = static_cast<float*>(e->x);
  float* q = static_cast<float*>(e->q);
  float* ao = static_cast<float*>(e->attn_o);
  float* act = static_cast<float*>(e->act);
  const float* wqkv = static_cast<const float*>(m.wqkv);
  const float* wo = static_cast<const float*>(m.wo);
  const float* wg = static_cast<const float*>(m.wgate);
  const float* wu = static_cast<const float*>(m.wup);
  const float* wd = static_cast<const float*>(m.wdown);
  DVLM_CK(f32_embed(static_cast<const float*>(m.embed), static_cast<const float*>(f.rows_in), f.n_src, f.tokens,
                    f.masked, m.mask_id, n, H, m.vocab, x, e->d_status, s));
  const int l1 = f.n_layers < 0 ? m.n_layers : f.layer0 + f.n_layers;
  const size_t kv_layer = static_cast<size_t>(Hkv) * e->Lmax * D;
  const double lb = std::log2(static_cast<double>(m.rope_base));
  for (int l = f.layer0; l < l1; ++l) {
    float* kc = static_cast<float*>(e->kc) + l * kv_layer;
    float* vc = static_cast<float*>(e->vc) + l * kv_layer;
    DVLM_CK(f32_rowscale(x, H, n, H, m.eps, e->f_r, s));
    DVLM_CK(f32_gemm(x, H, wqkv + static_cast<size_t>(l) * qkv_rows * H, qkv_rows, H, n, e->f_r, e->f_y, qkv_rows, s));
    DVLM_CK(f32_rope_scatter(e->f_y, n, Hq, Hkv, D, e->d_len, 0, lb, q, kc, vc, e->Lmax, s));
    DVLM_CK(f32_attention(q, ao, kc, vc, 1, n, f.n_clean, 0, e->d_len, e->Lmax, Hq, Hkv, D,
                          static_cast<float>(1.0 / std::sqrt(static_cast<double>(D))), s));
    DVLM_CK(f32_gemm(ao, Hq * D, wo + static_cast<size_t>(l) * H * Hq * D, H, Hq * D, n, nullptr, e->f_y, H, s));
    DVLM_CK(f32_add(x, H, e->f_y, H, n, H, s));
    DVLM_CK(f32_rowscale(x, H, n, H, m.eps, e->f_r, s));
    DVLM_CK(f32_gemm(x, H, wg + static_cast<size_t>(l) * I * H, I, H, n, e->f_r, e->f_g, I, s));
    DVLM_CK(f32_gemm(x, H, wu + static_cast<size_t>(l) * I * H, I, H, n, e->f_r, e->f_u, I, s));
    DVLM_CK(f32_swiglu(e->f_g, e->f_u, act, n * I, s));
    DVLM_CK(f32_gemm(act, I, wd + static_cast<size_t>(l) * H * I, H, I, n, nullptr, e->f_y, H, s));
    DVLM_CK(f32_add(x, H, e->f_y, H, n, H, s));
  }
  if (f.x_out) DVLM_CK(cudaMemcpyAsync(f.x_out, x, static_cast<size_t>(n) * H * 4, cudaMemcpyDeviceToDevice, s));
  if (f.lm) {
    LmArgs a = f.lma;
    fill_lm_scratch(e, a);
    DVLM_CK(f32_rowscale(x, H, n, H, m.eps, e->f_r, s));
    DVLM_CK(f32_lmhead(x, static_cast<const float*>(m.lm_head), a.R, H, m.vocab, e->f_r, e->f_p1, e->f_id, a, s));
  } else if (f.advance) {
    advance_kernel<<<1, 32, 0, s>>>(e->d_len, n);
    DVLM_CK(cudaGetLastError());
  }
  return cudaSuccess;
}

// Shapes the compute-bound prefill handles: 256-row weight tiles (two heads
// of 128 per QKV tile), 128-row gate/up tiles, k in 64-wide blocks.
bool prefill_gemm_supported(const dvlm_engine* e) {
  const dvlm_model& m = e->m;
  const int qkv_rows = (m.n_q_heads + 2 * m.n_kv_heads) * m.head_dim;
  return e->bf16 && !e->fp8 && !e->paged && e->max_ctx > 0 && m.head_dim == 128 && m.hidden % 256 == 0 && m.inter % 128 == 0 &&
         qkv_rows % 256 == 0 && (m.n_q_heads * m.head_dim) % 64 == 0;
}

// Prefill of n = n_vis + n_ids context rows at slots 0..n-1 [Fast-dVLM
// technical overview (ocdem.com), section 2.2.1: the exact KV cache of vision
// and prompt tokens the blocks attend to]: per layer one token-major GEMM per
// projection over all n rows and one causal attention launch; then the final
// norm and LM head of row n-1 give the first AR seed, and L = n.
cudaError_t engine_prefill_gemm(dvlm_engine* e, const void* vision, int n_vis, const int32_t* ids, int n_ids,
                                cudaStream_t s) {
  const dvlm_model& m = e->m;
  const int H = m.hidden, I = m.inter, D = m.head_dim, Hq = m.n_q_heads, Hkv = m.n_kv_heads;
  const int qkv_rows = (Hq + 2 * Hkv) * D;
  const int n = n_vis + n_ids, C = e->max_ctx;
  bf16* px = static_cast<bf16*>(e->px);
  DVLM_CK(cudaMemsetAsync(e->d_len, 0, 4, s));
  DVLM_CK(launch_embed_bf16(static_cast<const bf16*>(m.embed), static_cast<const bf16*>(vision), n_vis, ids, nullptr,
                            m.mask_id, n, H, m.vocab, px, e->pssq, C, e->d_status, false, s));
  // V^T as the attention reads it: keys past slot n - 1 are zero-filled by the
  // load (stale or poisoned cache slots never enter a product)
  CUtensorMap tm_vp;
  if (!make_tmap_2d(&tm_vp, e->vc, n, static_cast<uint64_t>(m.n_layers) * Hkv * D, static_cast<uint64_t>(e->Lmax) * 2,
                    64, 128))
    return cudaErrorInvalidValue;
  const size_t kv_layer = static_cast<size_t>(Hkv) * e->Lmax * D;
  TmArgs ta{};
  ta.n_tok = n;
  ta.tok_stride = C;
  ta.inv_h = 1.0f / H;
  ta.eps = m.eps;
  ta.Lmax = e->Lmax;
  ta.n_q_heads = Hq;
  ta.n_kv_heads = Hkv;
  ta.L0 = 0;
  ta.log2_rope_base = std::log2(static_cast<double>(m.rope_base));
  ta.status = e->d_status;
  ta.rope_cs = e->rope_cs;
  DVLM_CK(launch_rope_table(e->rope_cs, ta, s));
  PrefillAttnArgs pa{};
  pa.n_tok = n;
  pa.L0 = 0;
  pa.Lmax = e->Lmax;
  pa.Hq = Hq;
  pa.Hkv = Hkv;
  pa.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(D)));
  pa.out = static_cast<bf16*>(e->pao);
  pa.out_ld = Hq * D;
  pa.status = e->d_status;
  for (int l = 0; l < m.n_layers; ++l) {
    ta.epi = EPI_QKV;
    ta.ssq_in = e->pssq;
    ta.n_ssq = l == 0 ? H / 128 : H / 256;
    ta.out = static_cast<bf16*>(e->pq);
    ta.out_ld = Hq * D;
    ta.kcache = static_cast<bf16*>(e->kc) + l * kv_layer;
    ta.vcache = static_cast<bf16*>(e->vc) + l * kv_layer;
    DVLM_CK(launch_gemm_tm(e->tm_px, e->tm_wqkv_p, e->tm_wqkv_p, H / 64, l * qkv_rows, qkv_rows / 256, ta, s));
    pa.kv_base = l;
    DVLM_CK(launch_attn_prefill(e->tm_pq, e->tm_kp, tm_vp, pa, s));
    ta.epi = EPI_RESID;
    ta.resid = px;
    ta.resid_ld = H;
    ta.ssq_out = e->pssq;
    DVLM_CK(launch_gemm_tm(e->tm_pao, e->tm_wo_p, e->tm_wo_p, Hq * D / 64, l * H, H / 256, ta, s));
    ta.epi = EPI_SWIGLU;
    ta.n_ssq = H / 256;
    ta.out = static_cast<bf16*>(e->pact);
    ta.out_ld = I;
    DVLM_CK(launch_gemm_tm(e->tm_px, e->tm_wg_p, e->tm_wu_p, H / 64, l * I, I / 128, ta, s));
    ta.epi = EPI_RESID;
    DVLM_CK(launch_gemm_tm(e->tm_pact, e->tm_wd_p, e->tm_wd_p, I / 64, l * H, H / 256, ta, s));
  }
  // last context row -> decode buffer row 0 (with its sums of squares), then
  // the final norm + LM head: the AR seed of the first block, L = n
  DVLM_CK(launch_embed_bf16(nullptr, px + static_cast<size_t>(n - 1) * H, 1, nullptr, nullptr, 0, 1, H, m.vocab,
                            static_cast<bf16*>(e->x), e->ssq, kNT, e->d_status, false, s));
  LmArgs a{};
  a.R = 1;
  a.threshold = -1.0f;
  a.seed_out = e->d_seed;
  a.seed_row = 0;
  a.len_ptr = e->d_len;
  a.len_advance = n;
  fill_lm_scratch(e, a);
  a.ssq_in = e->ssq;
  a.n_ssq = H / 128;
  a.inv_h = 1.0f / H;
  a.eps = m.eps;
  const int nt = (m.vocab + 127) / 128;
  return launch_lmhead(kNT, e->tm_lm, e->tm_x, nt, H / 64, ws_ctas(e, static_cast<long long>(nt) * (H / 64)), a,
                       false, s);
}

// Split-K factor of a token-major GEMM with n_tiles output tiles and kb k
// blocks: enough CTAs to cover the SMs (all resident: the CTAs of a tile
// wait for one another), at least 4 k blocks each, at most `cap` (the tile's
// epilogue units: 16 for the residual epilogue, 8 otherwise).
static int tm_splits(const dvlm_engine* e, int n_tiles, int kb, int cap) {
  if (n_tiles >= e->sm) return 1;
  return std::max(1, std::min(cap, std::min(kb / 4, e->sm / n_tiles)));
}

bool quad_supported(const dvlm_engine* e, int B) {
  return prefill_gemm_supported(e) && B >= 1 && B <= 16 && B + B * B <= e->max_ctx &&
         e->m.n_q_heads == 8 * e->m.n_kv_heads;
}

// The fused forward of quadratic self-speculative decoding [Fast-dVLM
// technical overview (ocdem.com), section 2.3.1: draft and verify in one
// forward at O(B^2) cost] over the draft in e->tokens at slots L..L+B-1:
// B verify rows (causal; K/V to the cache) and B candidate blocks of B
// [MASK] rows (block i at positions L+i+1..; K/V to the side buffers, one
// layer at a time), all through the token-major GEMMs; the final residual
// rows end in e->px.  L is not advanced.
static cudaError_t quad_forward(dvlm_engine* e, int B, cudaStream_t s) {
  const dvlm_model& m = e->m;
  const int H = m.hidden, I = m.inter, D = m.head_dim, Hq = m.n_q_heads, Hkv = m.n_kv_heads;
  const int qkv_rows = (Hq + 2 * Hkv) * D;
  const int n = B + B * B, C = e->max_ctx;
  const int n_tt = (n + 127) / 128;
  bf16* px = static_cast<bf16*>(e->px);
  DVLM_CK(launch_quad_tokens(e->tokens, B, m.mask_id, e->qtok, s));
  DVLM_CK(launch_embed_bf16(static_cast<const bf16*>(m.embed), nullptr, 0, e->qtok, nullptr, m.mask_id, n, H,
                            m.vocab, px, e->pssq, C, e->d_status, false, s));
  const size_t kv_layer = static_cast<size_t>(Hkv) * e->Lmax * D;
  const float scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(D)));
  TmArgs ta{};
  ta.n_tok = n;
  ta.tok_stride = C;
  ta.inv_h = 1.0f / H;
  ta.eps = m.eps;
  ta.Lmax = e->Lmax;
  ta.n_q_heads = Hq;
  ta.n_kv_heads = Hkv;
  ta.d_len = e->d_len;
  ta.log2_rope_base = std::log2(static_cast<double>(m.rope_base));
  ta.status = e->d_status;
  ta.part = e->qpart;
  ta.cnt = e->qcnt;
  ta.quad_B = B;
  ta.kside = static_cast<bf16*>(e->kside);
  ta.vside = static_cast<bf16*>(e->vside);
  ta.side_n = kQuadSideKeys;
  ta.rope_cs = e->rope_cs;
  DVLM_CK(launch_rope_table(e->rope_cs, ta, s));
  AttnArgs aa{};
  aa.n_rows = B;
  aa.n_clean = B;
  aa.n_batch = 1;
  aa.d_len = e->d_len;
  aa.Lmax = e->Lmax;
  aa.Hq = Hq;
  aa.Hkv = Hkv;
  aa.scale_log2 = scale_log2;
  aa.out = static_cast<bf16*>(e->pao);
  aa.status = e->d_status;
  // candidate blocks: B batch entries of B noisy rows from row B on
  AttnArgs ac = aa;
  ac.n_clean = 0;
  ac.n_batch = B;
  ac.q_row0 = B;
  ac.cand_B = B;
  ac.side_n = kQuadSideKeys;
  // split-K factors (the residual epilogues leave (H / 256) * S sums of
  // squares per row for the next RMSNorm)
  const int s_qkv = tm_splits(e, n_tt * (qkv_rows / 256), H / 64, 8);
  const int s_o = tm_splits(e, n_tt * (H / 256), Hq * D / 64, 16);
  const int s_gu = tm_splits(e, n_tt * (I / 128), H / 64, 8);
  const int s_down = tm_splits(e, n_tt * (H / 256), I / 64, 16);
  for (int l = 0; l < m.n_layers; ++l) {
    ta.epi = EPI_QKV;
    ta.ssq_in = e->pssq;
    ta.n_ssq = l == 0 ? H / 128 : (H / 256) * s_down;
    ta.out = static_cast<bf16*>(e->pq);
    ta.out_ld = Hq * D;
    ta.kcache = static_cast<bf16*>(e->kc) + l * kv_layer;
    ta.vcache = static_cast<bf16*>(e->vc) + l * kv_layer;
    ta.splits = s_qkv;
    DVLM_CK(launch_gemm_tm(e->tm_px, e->tm_wqkv_p, e->tm_wqkv_p, H / 64, l * qkv_rows, qkv_rows / 256, ta, s));
    aa.kv_base = l;
    DVLM_CK(launch_attn_split_cl(e->tm_q3, e->tm_k, e->tm_v, aa, e->attn_cs, false, s));
    ac.kv_base = l;
    DVLM_CK(launch_attn_cand_cl(e->tm_q3, e->tm_k, e->tm_v, e->tm_ks, e->tm_vs, ac, e->attn_cs, s));
    ta.epi = EPI_RESID;
    ta.resid = px;
    ta.resid_ld = H;
    ta.ssq_out = e->pssq;
    ta.splits = s_o;
    DVLM_CK(launch_gemm_tm(e->tm_pao, e->tm_wo_p, e->tm_wo_p, Hq * D / 64, l * H, H / 256, ta, s));
    ta.epi = EPI_SWIGLU;
    ta.n_ssq = (H / 256) * s_o;
    ta.out = static_cast<bf16*>(e->pact);
    ta.out_ld = I;
    ta.splits = s_gu;
    DVLM_CK(launch_gemm_tm(e->tm_px, e->tm_wg_p, e->tm_wu_p, H / 64, l * I, I / 128, ta, s));
    ta.epi = EPI_RESID;
    ta.splits = s_down;
    DVLM_CK(launch_gemm_tm(e->tm_pact, e->tm_wd_p, e->tm_wd_p, I / 64, l * H, H / 256, ta, s));
  }
  return cudaSuccess;
}

// Trace records around an LM head the fused round runs directly.
static void quad_trace_begin(dvlm_engine* e, int kind, int n_rows, int n_clean, int R, const uint8_t* masked,
                             cudaStream_t s) {
  if (!e->trace_buf) return;
  trace_begin_kernel<<<1, 32, 0, s>>>(e->trace_buf, trace_record_bytes(e->m.hidden, e->bf16), e->trace_cap,
                                      e->trace_cnt, kind, e->d_len, n_rows, n_clean, R, e->tokens, masked);
}
static void quad_trace_end(dvlm_engine* e, int n_rows, int R, const uint8_t* masked, cudaStream_t s) {
  if (!e->trace_buf) return;
  trace_end_kernel<<<1, 256, 0, s>>>(e->trace_buf, trace_record_bytes(e->m.hidden, e->bf16), e->trace_cap,
                                     e->trace_cnt, e->d_len, e->d_seed, n_rows, R, e->tr_top1, e->tr_p1, e->tokens,
                                     masked, static_cast<const uint8_t*>(e->x),
                                     static_cast<size_t>(n_rows) * e->m.hidden * 2);
}

// One round of quadratic self-speculative decoding: the fused forward over
// the draft, the verify rows' LM head (row j predicts position j+1, L += B),
// the longest agreeing prefix k (L -= B - k, seed v_k, accepted tokens
// emitted), then the next draft: [v_k] followed by the top-1 of candidate
// block k-1's rows 0..B-2 (shift 1).
static cudaError_t quad_round(dvlm_engine* e, int B, int max_new, cudaStream_t s) {
  const dvlm_model& m = e->m;
  const int H = m.hidden;
  DVLM_CK(quad_forward(e, B, s));
  const int nt = (m.vocab + 127) / 128;
  const int lm_ctas = ws_ctas(e, static_cast<long long>(nt) * (H / 64));
  // verify rows -> decode rows (+ sums of squares), LM head over them
  DVLM_CK(launch_embed_bf16(nullptr, static_cast<const bf16*>(e->px), B, nullptr, nullptr, 0, B, H, m.vocab,
                            static_cast<bf16*>(e->x), e->ssq, kNT, e->d_status, false, s));
  quad_trace_begin(e, TR_QUAD_VERIFY, B, B, B, nullptr, s);
  LmArgs a{};
  a.R = B;
  a.threshold = -1.0f;
  a.id_out = e->vids + 1;
  a.len_ptr = e->d_len;
  a.len_advance = B;
  fill_lm_scratch(e, a);
  a.ssq_in = e->ssq;
  a.n_ssq = H / 128;
  a.inv_h = 1.0f / H;
  a.eps = m.eps;
  if (e->trace_buf) {
    a.top1_id = e->tr_top1;
    a.top1_prob = e->tr_p1;
  }
  DVLM_CK(launch_lmhead(kNT, e->tm_lm, e->tm_x, nt, H / 64, lm_ctas, a, false, s));
  quad_trace_end(e, B, B, nullptr, s);
  DVLM_CK(launch_decode_accept(e->vids, e->tokens, B, e->d_len, e->d_seed, e->stage_out, e->n_out, max_new, e->ahist,
                               e->d_k, e->d_status, false, s));
  // next draft from candidate block k-1
  DVLM_CK(launch_block_init(e->tokens, e->masked, e->d_seed, B, m.mask_id, 1, e->n_remaining, s));
  DVLM_CK(launch_select_cand_rows(static_cast<const bf16*>(e->px), H, e->d_k, B, static_cast<bf16*>(e->x), e->ssq,
                                  kNT, s));
  if (B > 1) {
    quad_trace_begin(e, TR_QUAD_CAND, B, 0, B - 1, e->masked, s);
    LmArgs c{};
    c.R = B - 1;
    c.masked = e->masked + 1;
    c.tokens = e->tokens + 1;
    c.threshold = -1.0f;  // the draft takes every position's argmax
    fill_lm_scratch(e, c);
    c.ssq_in = e->ssq;
    c.n_ssq = H / 128;
    c.inv_h = 1.0f / H;
    c.eps = m.eps;
    if (e->trace_buf) {
      c.top1_id = e->tr_top1;
      c.top1_prob = e->tr_p1;
    }
    DVLM_CK(launch_lmhead(kNT, e->tm_lm, e->tm_x, nt, H / 64, lm_ctas, c, false, s));
    quad_trace_end(e, B, B - 1, e->masked, s);
  }
  return cudaGetLastError();
}

// Test hook: the fused forward alone over the draft tokens (device [B]),
// its final residual rows [B + B*B][H] copied to x_out.
cudaError_t engine_forward_quad(dvlm_engine* e, const int32_t* draft, int B, void* x_out, cudaStream_t s) {
  DVLM_CK(cudaMemcpyAsync(e->tokens, draft, static_cast<size_t>(B) * 4, cudaMemcpyDeviceToDevice, s));
  DVLM_CK(quad_forward(e, B, s));
  return cudaMemcpyAsync(x_out, e->px, static_cast<size_t>(B + B * B) * e->m.hidden * 2, cudaMemcpyDeviceToDevice,
                         s);
}

cudaError_t engine_forward(dvlm_engine* e, const FwdSpec& f, cudaStream_t s) {
  return e->bf16 ? fwd_bf16(e, f, s) : fwd_f32(e, f, s);
}

// One forward of the decode driver, bracketed by the trace kernels when a
// trace buffer is set (the LM head then also reports its rows' ids and
// probabilities).  `tokens`/`masked` are the block state the trace records.
static cudaError_t traced_forward(dvlm_engine* e, FwdSpec f, int kind, const int32_t* tokens,
                                  const uint8_t* masked, cudaStream_t s) {
  if (!e->trace_buf) return engine_forward(e, f, s);
  const size_t rb = trace_record_bytes(e->m.hidden, e->bf16);
  trace_begin_kernel<<<1, 32, 0, s>>>(e->trace_buf, rb, e->trace_cap, e->trace_cnt, kind, e->d_len, f.n_rows,
                                      f.n_clean, f.lm ? f.lma.R : 0, tokens, masked);
  DVLM_CK(cudaGetLastError());
  // the LM head's per-row top-1 ids and probabilities are recorded from
  // where the forward puts them (a routing pass keeps them as anchors), or
  // from the trace's own buffers when the forward has no use for them
  if (f.lm) {
    if (!f.lma.top1_id) f.lma.top1_id = e->tr_top1;
    if (!f.lma.top1_prob) f.lma.top1_prob = e->tr_p1;
  }
  DVLM_CK(engine_forward(e, f, s));
  const size_t xb = static_cast<size_t>(f.n_rows) * e->m.hidden * (e->bf16 ? 2 : 4);
  trace_end_kernel<<<1, 256, 0, s>>>(e->trace_buf, rb, e->trace_cap, e->trace_cnt, e->d_len, e->d_seed, f.n_rows,
                                     f.lm ? f.lma.R : 0, f.lm ? f.lma.top1_id : e->tr_top1,
                                     f.lm ? f.lma.top1_prob : e->tr_p1, tokens, masked,
                                     static_cast<const uint8_t*>(e->x), xb);
  return cudaGetLastError();
}

// Replays the captured graph for `key`, capturing `body` on first use.
template <class F>
static cudaError_t run_graph(dvlm_engine* e, const std::vector<long long>& key, bool use_graphs, cudaStream_t s,
                             F&& body) {
  if (!use_graphs || s == nullptr) return body();
  auto it = e->graphs.find(key);
  if (it == e->graphs.end()) {
    DVLM_CK(cudaStreamBeginCapture(s, cudaStreamCaptureModeThreadLocal));
    const cudaError_t berr = body();
    cudaGraph_t g = nullptr;
    const cudaError_t cerr = cudaStreamEndCapture(s, &g);
    if (berr != cudaSuccess || cerr != cudaSuccess) {
      if (g) cudaGraphDestroy(g);
      return berr != cudaSuccess ? berr : cerr;
    }
    cudaGraphExec_t ex = nullptr;
    const cudaError_t ierr = cudaGraphInstantiate(&ex, g, 0);
    cudaGraphDestroy(g);
    DVLM_CK(ierr);
    it = e->graphs.emplace(key, ex).first;
  }
  return cudaGraphLaunch(it->second, s);
}

static long long fbits(float v) {
  uint32_t u;
  std::memcpy(&u, &v, 4);
  return u;
}

enum { G_NOISY = 1, G_APPEND, G_DRAFT, G_VERIFY, G_AR, G_QUAD, G_RFULL, G_RTEXT };

// One block (threshold / AR) or one round (spec).  Tokens are emitted into
// stage_out at n_out (capped at max_new).  Returns the number of tokens this
// step emitted, via *emitted (host).
cudaError_t engine_step(dvlm_engine* e, const dvlm_decode_cfg& cfg, int max_new, int n_out_host, int* emitted,
                        dvlm_stats* st, cudaStream_t s) {
  const int B = cfg.block_size;
  const bool ug = cfg.use_graphs != 0;
  if (cfg.mode == DVLM_MODE_AR) {
    DVLM_CK(run_graph(e, {G_AR, max_new}, ug, s, [&]() -> cudaError_t {
      FwdSpec f;
      f.tokens = e->d_seed;
      f.n_rows = 1;
      f.n_clean = 1;
      f.lm = true;
      f.lma.R = 1;
      f.lma.threshold = -1.0f;
      f.lma.seed_out = e->d_seed;
      f.lma.seed_row = 0;
      f.lma.len_ptr = e->d_len;
      f.lma.len_advance = 1;
      // emit the token being fed before the LM head overwrites the seed
      DVLM_CK(launch_emit(e->d_seed, 1, e->stage_out, e->n_out, max_new, false, s));
      return traced_forward(e, f, TR_AR, e->d_seed, nullptr, s);
    }));
    if (st) {
      st->nfe += 1;
      st->n_rounds += 1;
      st->n_launches += launches_per_forward(e->m.n_layers) + 1;
    }
    *emitted = std::min(1, max_new - n_out_host);
    return cudaSuccess;
  }
  auto draft_pass = [&]() -> cudaError_t {
    return run_graph(e, {G_DRAFT, B}, ug, s, [&]() -> cudaError_t {
      FwdSpec f;
      f.tokens = e->tokens;
      f.masked = e->masked;
      f.n_rows = B;
      f.n_clean = 0;
      f.lm = B > 1;
      f.lma.R = B - 1;
      f.lma.masked = e->masked + 1;
      f.lma.tokens = e->tokens + 1;
      f.lma.threshold = -1.0f;  // the draft takes every position's argmax
      return traced_forward(e, f, TR_DRAFT, e->tokens, e->masked, s);
    });
  };
  if (cfg.mode == DVLM_MODE_SPEC_QUAD) {
    // quadratic self-speculative round [Fast-dVLM technical overview
    // (ocdem.com), section 2.3.1]: the first round of a run drafts with one
    // diffusion pass; every round is then one fused draft+verify forward
    if (!e->quad_ready || e->quad_B != B) {
      DVLM_CK(launch_block_init(e->tokens, e->masked, e->d_seed, B, e->m.mask_id, 1, e->n_remaining, s));
      DVLM_CK(draft_pass());
      e->quad_ready = true;
      e->quad_B = B;
      if (st) {
        st->nfe += 1;
        st->n_launches += 1 + (B > 1 ? 1 : 0) * launches_per_forward(e->m.n_layers);
      }
    }
    DVLM_CK(run_graph(e, {G_QUAD, B, max_new}, ug, s, [&]() { return quad_round(e, B, max_new, s); }));
    int32_t h = 0;
    DVLM_CK(cudaMemcpyAsync(&h, e->n_out, 4, cudaMemcpyDeviceToHost, s));
    DVLM_CK(cudaStreamSynchronize(s));
    if (h <= n_out_host) return cudaErrorLaunchTimeout;
    if (st) {
      st->nfe += 1;
      st->n_rounds += 1;
      st->n_launches += 8 + 6 * e->m.n_layers + (B > 1 ? 1 : 0);
    }
    *emitted = h - n_out_host;
    return cudaSuccess;
  }
  DVLM_CK(launch_block_init(e->tokens, e->masked, e->d_seed, B, e->m.mask_id, 1, e->n_remaining, s));
  if (cfg.mode == DVLM_MODE_ROUTE || cfg.mode == DVLM_MODE_THRESHOLD) {
  if (cfg.mode == DVLM_MODE_ROUTE) {
    // certificate-guided visual routing [Look Only When Needed, method
    // steps (1)-(3)]; position j is scored by row j-1 (rows 0..B-2)
    const int k = cfg.route_k, nv = cfg.route_n_vis;
    int n_masked = B - 1;
    bool have_anchors = false;
    for (int step = 0; n_masked > 0; ++step) {
      // every step unmasks at least one position
      if (step >= 2 * (B - 1)) return cudaErrorLaunchTimeout;
      const int kk = std::min(k, n_masked);
      if (have_anchors) {
        DVLM_CK(run_graph(e, {G_RTEXT, B, nv}, ug, s, [&]() -> cudaError_t {
          FwdSpec f;
          f.tokens = e->tokens;
          f.masked = e->masked;
          f.n_rows = B;
          f.n_clean = 0;
          f.hide = nv;
          f.lm = true;
          f.lma.R = B - 1;
          f.lma.masked = e->masked + 1;
          f.lma.threshold = 2.0f;
          f.lma.top1_id = e->txt_id;
          f.lma.top1_prob = e->txt_p1;
          f.lma.anchor_id = e->anc_id;
          f.lma.anchor_conf = e->anc_p1;
          f.lma.cert_len = e->cert;
          return traced_forward(e, f, TR_ROUTE_TEXT, e->tokens, e->masked, s);
        }));
        int32_t cert = 0;
        DVLM_CK(cudaMemcpyAsync(&cert, e->cert, 4, cudaMemcpyDeviceToHost, s));
        DVLM_CK(cudaStreamSynchronize(s));
        if (st) {
          st->nfe += 1;
          st->n_iters += 1;
          st->n_text_passes += 1;
          st->n_launches += launches_per_forward(e->m.n_layers);
        }
        if (cert >= kk) {  // the certified prefix, with the anchor ids
          DVLM_CK(launch_topk_commit(e->anc_p1, e->anc_id, nullptr, e->masked + 1, e->tokens + 1, B - 1, cert,
                                     nullptr, nullptr, s));
          n_masked -= cert;
          if (st && cert < DVLM_HIST) st->commit_hist[cert] += 1;
          continue;
        }
      }
      DVLM_CK(run_graph(e, {G_RFULL, B}, ug, s, [&]() -> cudaError_t {
        FwdSpec f;
        f.tokens = e->tokens;
        f.masked = e->masked;
        f.n_rows = B;
        f.n_clean = 0;
        f.lm = true;
        f.lma.R = B - 1;
        f.lma.masked = e->masked + 1;
        f.lma.threshold = 2.0f;
        f.lma.top1_id = e->anc_id;  // the FULL pass replaces every anchor
        f.lma.top1_prob = e->anc_p1;
        return traced_forward(e, f, TR_ROUTE_FULL, e->tokens, e->masked, s);
      }));
      DVLM_CK(launch_topk_commit(e->anc_p1, e->anc_id, have_anchors ? e->txt_id : nullptr, e->masked + 1,
                                 e->tokens + 1, B - 1, kk, nullptr, nullptr, s));
      n_masked -= kk;
      have_anchors = true;
      if (st) {
        st->nfe += 1;
        st->n_iters += 1;
        st->n_launches += launches_per_forward(e->m.n_layers) + 1;
        if (kk < DVLM_HIST) st->commit_hist[kk] += 1;
      }
    }
  } else {
    int rem = B - 1;
    for (int it = 0; rem > 0; ++it) {
      // every iteration commits at least one position: a block needing more
      // than B - 1 means a device-side wait gave up (see the status word)
      if (it >= B - 1) return cudaErrorLaunchTimeout;
      DVLM_CK(run_graph(e, {G_NOISY, B, fbits(cfg.threshold)}, ug, s, [&]() -> cudaError_t {
        FwdSpec f;
        f.tokens = e->tokens;
        f.masked = e->masked;
        f.n_rows = B;
        f.n_clean = 0;
        f.lm = true;
        // position j is scored by row j-1: rows 0..B-2 commit into positions 1..B-1
        f.lma.R = B - 1;
        f.lma.masked = e->masked + 1;
        f.lma.tokens = e->tokens + 1;
        f.lma.threshold = cfg.threshold;
        f.lma.n_remaining = e->n_remaining;
        f.lma.hist = e->hist;
        return traced_forward(e, f, TR_NOISY, e->tokens, e->masked, s);
      }));
      int32_t h = 0;
      DVLM_CK(cudaMemcpyAsync(&h, e->n_remaining, 4, cudaMemcpyDeviceToHost, s));
      DVLM_CK(cudaStreamSynchronize(s));
      rem = h;
      if (st) {
        st->nfe += 1;
        st->n_iters += 1;
        st->n_launches += launches_per_forward(e->m.n_layers);
      }
    }
  }
    DVLM_CK(run_graph(e, {G_APPEND, B, max_new}, ug, s, [&]() -> cudaError_t {
      FwdSpec f;
      f.tokens = e->tokens;
      f.n_rows = B;
      f.n_clean = B;
      f.lm = true;
      f.lma.R = B;
      f.lma.threshold = -1.0f;
      f.lma.seed_out = e->d_seed;
      f.lma.seed_row = B - 1;
      f.lma.len_ptr = e->d_len;
      f.lma.len_advance = B;
      DVLM_CK(traced_forward(e, f, TR_APPEND, e->tokens, nullptr, s));
      return launch_emit(e->tokens, B, e->stage_out, e->n_out, max_new, true, s);
    }));
    if (st) {
      st->nfe += 1;
      st->n_rounds += 1;
      st->n_launches += launches_per_forward(e->m.n_layers) + 2;  // + block init + emit
    }
    *emitted = std::min(B, max_new - n_out_host);
    return cudaSuccess;
  }
  // linear self-speculative round
  DVLM_CK(draft_pass());
  DVLM_CK(run_graph(e, {G_VERIFY, B, max_new}, ug, s, [&]() -> cudaError_t {
    FwdSpec f;
    f.tokens = e->tokens;
    f.n_rows = B;
    f.n_clean = B;
    f.lm = true;
    f.lma.R = B;
    f.lma.threshold = -1.0f;
    f.lma.id_out = e->vids + 1;  // row j predicts position j+1
    f.lma.len_ptr = e->d_len;
    f.lma.len_advance = B;
    DVLM_CK(traced_forward(e, f, TR_VERIFY, e->tokens, nullptr, s));
    return launch_decode_accept(e->vids, e->tokens, B, e->d_len, e->d_seed, e->stage_out, e->n_out, max_new,
                                e->ahist, nullptr, e->d_status, true, s);
  }));
  int32_t h = 0;
  DVLM_CK(cudaMemcpyAsync(&h, e->n_out, 4, cudaMemcpyDeviceToHost, s));
  DVLM_CK(cudaStreamSynchronize(s));
  // a round always keeps at least the AR seed: none means a device-side wait gave up
  if (h <= n_out_host) return cudaErrorLaunchTimeout;
  if (st) {
    st->nfe += 2;
    st->n_rounds += 1;
    st->n_launches += 2 + (B > 1 ? 2 : 1) * launches_per_forward(e->m.n_layers);  // + block init + accept
  }
  *emitted = h - n_out_host;
  return cudaSuccess;
}

cudaError_t engine_collect_stats(dvlm_engine* e, dvlm_stats* st, cudaStream_t s) {
  int64_t h[2 * DVLM_HIST];
  DVLM_CK(cudaMemcpyAsync(h, e->hist, DVLM_HIST * 8, cudaMemcpyDeviceToHost, s));
  DVLM_CK(cudaMemcpyAsync(h + DVLM_HIST, e->ahist, DVLM_HIST * 8, cudaMemcpyDeviceToHost, s));
  DVLM_CK(cudaStreamSynchronize(s));
  if (st) {
    for (int i = 0; i < DVLM_HIST; ++i) {
      st->commit_hist[i] += h[i];
      st->accept_hist[i] += h[DVLM_HIST + i];
    }
  }
  DVLM_CK(cudaMemsetAsync(e->hist, 0, DVLM_HIST * 8, s));
  return cudaMemsetAsync(e->ahist, 0, DVLM_HIST * 8, s);
}

// One eager forward with CUDA events around every kernel: per-kind device
// time (ms, summed over layers) and launch counts.
cudaError_t engine_profile(dvlm_engine* e, const FwdSpec& f0, float* ms, int* counts, cudaStream_t s) {
  KernelTimer tm;
  tm.s = s;
  FwdSpec f = f0;
  f.timer = &tm;
  cudaError_t err = engine_forward(e, f, s);
  if (err == cudaSuccess) err = cudaStreamSynchronize(s);
  for (int k = 0; k < K_KINDS; ++k) {
    ms[k] = 0.f;
    counts[k] = 0;
  }
  for (auto& mk : tm.marks) {
    float t = 0.f;
    if (err == cudaSuccess) err = cudaEventElapsedTime(&t, mk.second.first, mk.second.second);
    ms[mk.first] += t;
    counts[mk.first] += 1;
    cudaEventDestroy(mk.second.first);
    cudaEventDestroy(mk.second.second);
  }
  return err;
}

// Tuning knobs (cluster sizes, pipeline depths, PDL); invalidates captured graphs.
dvlm_status engine_set_option(dvlm_engine* e, const char* name, int v) {
  const dvlm_model& m = e->m;
  const std::string n(name);
  if (e->fp8 && n != "pdl" && n != "attn_cluster" && n != "attn_split") return DVLM_ERR_UNSUPPORTED;
  // every cluster of the projection resident at once (one wave)
  const int qkv_tiles = (m.n_q_heads + 2 * m.n_kv_heads) * m.head_dim / 128, h_tiles = m.hidden / 128;
  auto cluster_ok = [&](int epi, int S, int stages, int n_tiles) {
    return S == 0 || (S >= 2 && S <= 16 && gemm_cl_max_clusters(epi, S, stages) >= n_tiles);
  };
  if (n == "qkv_cluster") {
    if (!cluster_ok(EPI_QKV, v, 5, qkv_tiles) || v > m.hidden / 64) return DVLM_ERR_UNSUPPORTED;
    e->s_qkv = v;
  } else if (n == "o_cluster") {
    if (!cluster_ok(EPI_RESID, v, 5, h_tiles) || v > m.n_q_heads * m.head_dim / 64) return DVLM_ERR_UNSUPPORTED;
    e->s_o = v;
  } else if (n == "down_cluster") {
    if (!cluster_ok(EPI_RESID, v, e->down_stages, h_tiles) || v > m.inter / 64) return DVLM_ERR_UNSUPPORTED;
    e->s_down = v;
  } else if (n == "down_stages") {
    if (v != 5 && v != 10) return DVLM_ERR_SHAPE;
    if (!cluster_ok(EPI_RESID, e->s_down, v, h_tiles)) return DVLM_ERR_UNSUPPORTED;
    // 5-stage down CTAs fit beside 5-stage gate/up CTAs: launched early, they
    // could take the room of gate/up CTAs not yet resident, whose stream-K
    // partials the resident ones wait for (the wait would run out)
    if (v == 5 && e->gu_stages == 5) return DVLM_ERR_UNSUPPORTED;
    e->down_stages = v;
  } else if (n == "gateup_stages") {
    if (v != 5 && v != 10) return DVLM_ERR_SHAPE;
    if (v == 10 && e->gu_cps == 2) return DVLM_ERR_UNSUPPORTED;
    if (v == 5 && e->down_stages == 5) return DVLM_ERR_UNSUPPORTED;  // see "down_stages"
    e->gu_stages = v;
  } else if (n == "gateup_ctas_per_sm") {
    if (v != 1 && v != 2) return DVLM_ERR_SHAPE;
    if (v == 2 && e->gu_stages == 10) return DVLM_ERR_UNSUPPORTED;
    e->gu_cps = v;
  } else if (n == "attn_cluster") {
    if (v != 8 && v != 16) return DVLM_ERR_SHAPE;
    if (attn_split_cl_max_clusters(v) <= 0) return DVLM_ERR_UNSUPPORTED;
    e->attn_cs = v;
  } else if (n == "pdl") {
    e->pdl = v != 0;
  } else if (n == "attn_split") {
    if (v < 0 || v > kMaxAttnSplit) return DVLM_ERR_SHAPE;
    e->attn_split = v;
  } else if (n == "persistent") {
    if (v != 0 && v != 1) return DVLM_ERR_SHAPE;
    if (v && !persistent_supported(e)) return DVLM_ERR_UNSUPPORTED;
    e->chain = v != 0;
  } else if (n == "prefill_gemm") {
    if (v != 0 && v != 1) return DVLM_ERR_SHAPE;
    if (v && !prefill_gemm_supported(e)) return DVLM_ERR_UNSUPPORTED;
    e->prefill_gemm = v != 0;
  } else {
    return DVLM_ERR_INVALID_ARG;
  }
  for (auto& kv : e->graphs) cudaGraphExecDestroy(kv.second);
  e->graphs.clear();
  return DVLM_OK;
}

int engine_get_option(dvlm_engine* e, const char* name) {
  const std::string n(name);
  if (n == "qkv_cluster") return e->s_qkv;
  if (n == "o_cluster") return e->s_o;
  if (n == "down_cluster") return e->s_down;
  if (n == "down_stages") return e->down_stages;
  if (n == "gateup_stages") return e->gu_stages;
  if (n == "gateup_ctas_per_sm") return e->gu_cps;
  if (n == "attn_cluster") return e->attn_cs;
  if (n == "pdl") return e->pdl ? 1 : 0;
  if (n == "attn_split") return e->attn_split;
  if (n == "prefill_gemm") return e->prefill_gemm ? 1 : 0;
  if (n == "persistent") return e->chain ? 1 : 0;
  return -1;
}

// Sets (or clears, buf == NULL) the forward trace; captured graphs are
// rebuilt with or without the trace kernels.
void engine_set_trace(dvlm_engine* e, void* buf, int cap, int32_t* cnt) {
  e->trace_buf = static_cast<uint8_t*>(buf);
  e->trace_cap = buf ? cap : 0;
  e->trace_cnt = buf ? cnt : nullptr;
  for (auto& kv : e->graphs) cudaGraphExecDestroy(kv.second);
  e->graphs.clear();
}

// Switches the engine to a paged KV cache [Fast-dVLM technical overview
// (ocdem.com), section 2.3.2: paged KV cache management]: attention reads
// 64-key chunks through the block table, the QKV epilogue writes each new
// K/V row through it; the compute-bound prefill, the fused quadratic forward
// and the TEXT-ONLY views (contiguous layouts) are not used.
bool engine_set_paged(dvlm_engine* e, void* k_pages, void* v_pages, const int32_t* table, int n_pages,
                      int max_pages) {
  const dvlm_model& m = e->m;
  const uint64_t rows = static_cast<uint64_t>(m.n_layers) * n_pages * m.n_kv_heads;
  CUtensorMap tk, tv;
  if (!make_tmap_2d(&tk, k_pages, m.head_dim, rows * 64, m.head_dim * 2, 64, 64) ||
      !make_tmap_2d(&tv, v_pages, 64, rows * m.head_dim, 64 * 2, 64, 128))
    return false;
  e->tm_k = tk;
  e->tm_v = tv;
  e->kc = k_pages;
  e->vc = v_pages;
  e->block_table = table;
  e->n_pages = n_pages;
  e->max_pages = max_pages;
  e->paged = true;
  e->prefill_gemm = false;
  e->quad_ready = false;
  for (auto& kv : e->graphs) cudaGraphExecDestroy(kv.second);
  e->graphs.clear();
  return true;
}

size_t engine_workspace_bytes(dvlm_engine* e, int P) { return carve(e, nullptr, true, P); }
size_t engine_carve(dvlm_engine* e, void* ws, int P) { return carve(e, static_cast<uint8_t*>(ws), false, P); }
bool engine_build_maps(dvlm_engine* e) { return build_maps(e); }

// Cluster size for a projection with n_tiles output tiles: the largest S with
// n_tiles * S <= SMs whose clusters can all be resident at once (0: use the
// stream-K kernel instead).
static int pick_cluster(dvlm_engine* e, int epi, int n_tiles, int kb, int stages) {
  for (int S = std::min(16, std::min(kb, e->sm / std::max(1, n_tiles))); S >= 2; --S)
    if (gemm_cl_max_clusters(epi, S, stages) >= n_tiles) return S;
  return 0;
}

// Same for the W8A8 kernels (kb = 128-wide k blocks; each CTA's share of them
// must fit its activation-code buffer of 16 blocks).
static int pick_cluster_fp8(dvlm_engine* e, int epi, int n_tiles, int kb, int stages) {
  for (int S = std::min(16, std::min(kb, e->sm / std::max(1, n_tiles))); S >= 2; --S)
    if ((kb + S - 1) / S <= 16 && gemm_cl_max_clusters_fp8(epi, S, stages) >= n_tiles) return S;
  return 0;
}

void engine_plan(dvlm_engine* e) {
  if (!e->bf16) return;
  const dvlm_model& m = e->m;
  const int qkv_rows = (m.n_q_heads + 2 * m.n_kv_heads) * m.head_dim;
  if (e->fp8) {
    e->s_qkv = pick_cluster_fp8(e, EPI_QKV, qkv_rows / 128, m.hidden / 128, 5);
    e->s_o = pick_cluster_fp8(e, EPI_RESID, m.hidden / 128, m.n_q_heads * m.head_dim / 128, 5);
    e->s_down = pick_cluster_fp8(e, EPI_RESID, m.hidden / 128, m.inter / 128, e->down_stages);
    e->attn_cs = attn_split_cl_max_clusters(16) >= m.n_kv_heads ? 16 : 8;
    e->prefill_gemm = false;
    return;
  }
  e->s_qkv = pick_cluster(e, EPI_QKV, qkv_rows / 128, m.hidden / 64, 5);
  e->s_o = pick_cluster(e, EPI_RESID, m.hidden / 128, m.n_q_heads * m.head_dim / 64, 5);
  e->s_down = pick_cluster(e, EPI_RESID, m.hidden / 128, m.inter / 64, e->down_stages);
  // 16-CTA attention clusters when one per KV head can be resident at once
  e->attn_cs = attn_split_cl_max_clusters(16) >= m.n_kv_heads ? 16 : 8;
  e->prefill_gemm = prefill_gemm_supported(e);
}

}  // namespace dvlm
