// Internal launch interface between the C-ABI/engine layer and the kernels.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "dvlm.h"

namespace dvlm {

using bf16 = __nv_bfloat16;

enum EpiKind { EPI_QKV = 0, EPI_RESID = 1, EPI_SWIGLU = 2 };

// Fused-epilogue operands of the decoder GEMMs.
struct GemmEpi {
  int epi;
  int n_rows;                 // valid token rows (<= NT)
  // RMSNorm factor of the input rows, from per-128-feature sums of squares
  const float* ssq_in;        // [n_ssq][NT]
  int n_ssq;
  float inv_h, eps;
  // EPI_QKV: q [rows][Hq*D]; EPI_SWIGLU: act [rows][I]
  bf16* out;
  int out_ld;
  // EPI_RESID: residual stream [rows][H] updated in place, ssq_out [n_tiles][NT]
  bf16* resid;
  int resid_ld;
  float* ssq_out;
  // EPI_QKV: KV cache of this layer; K [Hkv][Lmax][D], V^T [Hkv][D][Lmax]
  bf16* kcache;
  bf16* vcache;
  int Lmax, n_q_heads, n_kv_heads;
  const int* d_len;           // slot of row 0 (device); NULL -> L_static
  int L_static;
  double log2_rope_base;
  // stream-K scratch: part [P][NT][128] fp32 (one partial tile per CTA), cnt [n_tiles] int (zero)
  float* part;
  int* cnt;
  int* status;
  // W8A8 (fp8 kernels only): the projection's input rows q_src [NT][q_ld]
  // (K wide; with rms_input the projection consumes their RMSNorm) are
  // quantised per token in the CTA; amax_in [n_amax][NT] gives their largest
  // magnitudes (else the rows are scanned); wscale / wscale2 are the E4M3
  // weights' per-row scales indexed by absolute weight row (wscale2: the up
  // rows of gate/up tiles); amax_out [n_tiles][NT] receives the SwiGLU
  // activation's largest magnitude per tile (the down projection's amax_in).
  const bf16* q_src;
  int q_ld, q_K, rms_input;
  const float* amax_in;
  int n_amax;
  const float* wscale;
  const float* wscale2;
  float* amax_out;
  // Paged cache (block_table != NULL): slot s of the sequence is row s % 64 of
  // page block_table[s / 64] (n_pages pages); kcache / vcache then point at
  // this layer's pages, K [n_pages][Hkv][64][128], V^T [n_pages][Hkv][128][64].
  const int* block_table;
  int n_pages;
};

// Destination of cache slot `slot`, KV head h (value feature j) in a
// contiguous or paged cache (see GemmEpi); NULL for a page id out of range.
__device__ __forceinline__ bf16* kv_k_ptr(const GemmEpi& ea, int h, int slot) {
  if (!ea.block_table) return ea.kcache + (static_cast<size_t>(h) * ea.Lmax + slot) * 128;
  const int page = ea.block_table[slot >> 6];
  if (page < 0 || page >= ea.n_pages) return nullptr;
  return ea.kcache + (static_cast<size_t>(page * ea.n_kv_heads + h) * 64 + (slot & 63)) * 128;
}
__device__ __forceinline__ bf16* kv_v_ptr(const GemmEpi& ea, int h, int j, int slot) {
  if (!ea.block_table) return ea.vcache + (static_cast<size_t>(h) * 128 + j) * ea.Lmax + slot;
  const int page = ea.block_table[slot >> 6];
  if (page < 0 || page >= ea.n_pages) return nullptr;
  return ea.vcache + (static_cast<size_t>(page * ea.n_kv_heads + h) * 128 + j) * 64 + (slot & 63);
}

// Fused LM head operands.
struct LmArgs {
  int R;                     // rows to report/commit (<= NT)
  int V;
  const float* ssq_in;       // final RMSNorm sums of squares [n_ssq][NT] or NULL
  int n_ssq;
  float inv_h, eps;
  // scratch
  float* part;               // [P][NT][128] partial logits of split tiles
  int* cnt;                  // [n_tiles] (zero between launches)
  float* rec;                // [P][NT][4]: per-CTA (m, s, idx)
  int* done;                 // [1] (zero between launches)
  // commit / outputs
  uint8_t* masked;
  int32_t* tokens;
  float threshold;
  int32_t* top1_id;
  float* top1_prob;
  uint8_t* commit;
  int32_t* n_commit;
  const int32_t* anchor_id;
  const float* anchor_conf;
  int32_t* cert_len;
  int32_t* n_remaining;      // masked rows left after the commit
  int32_t* len_ptr;          // *len_ptr += len_advance at the end (may be NULL)
  int len_advance;
  int32_t* seed_out;         // *seed_out = top1_id[seed_row] (may be NULL)
  int seed_row;
  int32_t* id_out;           // id_out[r] = top1_id[r] for r < R (may be NULL)
  int64_t* hist;             // commit histogram (may be NULL)
  int64_t* nfe;              // +1 per call (may be NULL)
  int* status;
};

struct Launch {
  int sm_count;
  bool pdl;
};

int device_sm_count();
// stages: 5 (two CTAs per SM) or 10 (one CTA per SM, deeper stream) for NT=16; 4 for NT=32.
cudaError_t launch_gemm_ws(int NT, const CUtensorMap& mapA, const CUtensorMap& mapA2, const CUtensorMap& mapB,
                           int n_tiles, int kb, int P, int a_row_base, const GemmEpi& ea, bool pdl, cudaStream_t s,
                           int stages);
// W8A8 variants (E4M3 weight maps with 128-byte k boxes; kb = K / 128): the
// stream-K gate/up kernel (10 stages) and the cluster split-K kernels.
cudaError_t launch_gemm_ws_fp8(const CUtensorMap& mapA, const CUtensorMap& mapA2, int n_tiles, int kb, int P,
                               int a_row_base, const GemmEpi& ea, bool pdl, cudaStream_t s);
cudaError_t launch_gemm_cl_fp8(const CUtensorMap& mapA, int n_tiles, int kb, int S, int a_row_base, const GemmEpi& ea,
                               bool pdl, cudaStream_t s, int stages);
int gemm_cl_max_clusters_fp8(int epi, int S, int stages);
size_t gemm_ws_part_bytes(int NT, int P);
// Cluster split-K (one tile per cluster of S CTAs; QKV and residual epilogues).
cudaError_t launch_gemm_cl(int NT, const CUtensorMap& mapA, const CUtensorMap& mapB, int n_tiles, int kb, int S,
                           int a_row_base, const GemmEpi& ea, bool pdl, cudaStream_t s, int stages);
int gemm_cl_max_clusters(int epi, int S, int stages);

// Persistent forward (bf16 weights, 16 token rows): every decoder layer of
// one forward in a single launch of one CTA per SM, phase by phase -- the
// first layer's QKV, then per layer l: attention partials, attention merge,
// O-projection, gate/up, down, and QKV of layer l+1 (not after the last
// layer) -- with a grid barrier between phases.  The four GEMM phases are
// given in their first-layer form: weight rows of layer l start at
// l * (qkv_rows | H | I | H); the QKV phase's cache pointers move by
// kv_layer elements per layer.  Each GEMM phase's ea.cnt is its own block of
// n_tiles zeroed ints; ea.part holds one partial tile per CTA.
struct ChainPhase {
  CUtensorMap mapA, mapA2, mapB;
  GemmEpi ea;
  int n_tiles, kb, a_row_base;
  int ctas;  // CTAs that stream the phase (at most the grid): fewer for the narrow products, so that
             // their split tiles have fewer parts to add (their weights are prefetched anyway)
};
struct FwdProgram {
  ChainPhase qkv, o, gu, down;
  int qkv_rows, H, I;
  size_t kv_layer;
  // attention: q [16][Hq][128] (3-D map, 64 x 8 x 16 box), the cache's K
  // rows ((layer * Hkv + g) * Lmax + slot, 64 x 64 box) and V^T rows
  // ((layer * Hkv + g) * 128 + d, 64-key x 128 box); Hq = 8 * Hkv
  CUtensorMap mapQ, mapK, mapV;
  int Hq, Hkv, Lmax, n_clean;
  float scale_log2;
  float* apart;   // [Hkv][n_chunks_max][128 features][128 rows] unnormalised partial rows (fp32)
  float2* aml;    // [Hkv][n_chunks_max][128 rows] (row max, row sum) per 64-key chunk
  int n_chunks_max;
  bf16* attn_o;   // [16][Hq * 128] merged attention rows, the O-projection's input
  int layer0, n_layers;
  int* bar;       // [2] barrier and exit counters: zero before the first launch, zero again after each
  int* status;
};
cudaError_t launch_fwd_persistent(const FwdProgram& fp, int P, bool pdl, cudaStream_t s);
// CTAs of the persistent forward that can be resident at once on the current device (0 on error).
int fwd_persistent_max_ctas();
// Scratch of the attention phases for caches of Lmax slots: apart, then aml.
size_t fwd_attn_scratch_bytes(int Hkv, int Lmax);
cudaError_t launch_lmhead(int NT, const CUtensorMap& mapW, const CUtensorMap& mapH, int n_tiles, int kb, int P,
                          const LmArgs& a, bool pdl, cudaStream_t s);
size_t lmhead_scratch_bytes(int NT, int P, int n_tiles);

// Attention over the KV cache (bf16 tcgen05 path).
struct AttnArgs {
  int n_rows, n_clean, n_batch;
  int L_static;
  const int* d_len;
  int Lmax, Hq, Hkv;
  int kv_base;               // cache entry of batch 0 (the layer, in the engine)
  float scale_log2;          // scale * log2(e)
  bf16* out;                 // [n_batch][n_rows][Hq][128]
  int* status;
  int len_sub;               // the length used is (*d_len or L_static) - len_sub (offset cache views)
  // Paged cache (block_table != NULL): 64-slot pages; logical slot s of batch
  // entry b lives in row s % 64 of page block_table[b * max_pages + s / 64].
  // K pages [kv_base layers][n_pages][Hkv][64][128], V^T pages
  // [layers][n_pages][Hkv][128][64]; d_lens[b] (device) is entry b's length.
  const int* block_table;
  int max_pages, n_pages;
  const int* d_lens;
  // Queries and outputs start at row q_row0 of their buffers (batch entry b's
  // rows at q_row0 + b * n_rows).
  int q_row0;
  // Candidate blocks of a fused draft+verify forward (cand_B = B > 0,
  // launch_attn_cand_cl): batch entry b is candidate block b, B noisy rows
  // that see the cache slots 0..*d_len + b (the context and the first b + 1
  // draft tokens) and the block's own B keys, side_n-key rows of the side
  // buffers (K [Hkv][side_n][128], V^T [Hkv][128][side_n]) from key b * 64.
  int cand_B, side_n;
};
// Block attention (csrc/attn_split.cu), two forms of one kernel.  Split form:
// S independent CTAs per (batch entry, 16-row group, KV head), merged by the
// last to finish; scratch of attn_split_scratch_bytes(n_batch * n_groups *
// Hkv, S) bytes whose counters start at zero (they are zero again after each
// launch).
size_t attn_split_scratch_bytes(int n_groups_total, int S);
cudaError_t launch_attn_split(const CUtensorMap& mapQ, const CUtensorMap& mapK, const CUtensorMap& mapV,
                              const AttnArgs& a, int S, void* scratch, bool pdl, cudaStream_t s);
// Cluster form (the decode path): the S = cs splits of a group are one
// thread-block cluster (cs = 8, or 16 where two 16-CTA clusters can be
// resident at once: attn_split_cl_max_clusters), merged through distributed
// shared memory; no scratch.
cudaError_t launch_attn_split_cl(const CUtensorMap& mapQ, const CUtensorMap& mapK, const CUtensorMap& mapV,
                                 const AttnArgs& a, int cs, bool pdl, cudaStream_t s);
// Cluster form over the candidate blocks (a.cand_B > 0); mapKs / mapVs: the
// side buffers with the boxes of mapK / mapV.
cudaError_t launch_attn_cand_cl(const CUtensorMap& mapQ, const CUtensorMap& mapK, const CUtensorMap& mapV,
                                const CUtensorMap& mapKs, const CUtensorMap& mapVs, const AttnArgs& a, int cs,
                                cudaStream_t s);
int attn_split_cl_max_clusters(int cs);

// Prefill (compute-bound path over the whole context; csrc/prefill.cu).
// Token-major GEMM epilogue operands: one context row per epilogue thread.
struct TmArgs {
  int epi;
  int n_tok;                  // valid context rows
  int tok_stride;             // ssq arrays are [entry][tok_stride]
  const float* ssq_in;        // RMSNorm input sums of squares (QKV, SWIGLU)
  int n_ssq;
  float inv_h, eps;
  bf16* out;                  // QKV: q [n_tok][Hq*128]; SWIGLU: act [n_tok][I]
  int out_ld;
  bf16* resid;                // RESID: residual stream [n_tok][H], updated in place
  int resid_ld;
  float* ssq_out;             // RESID: [H/256][tok_stride]
  bf16* kcache;               // QKV: this layer's K [Hkv][Lmax][128] and V^T [Hkv][128][Lmax]
  bf16* vcache;
  int Lmax, n_q_heads, n_kv_heads;
  int L0;                     // cache slot of context row 0 (d_len != NULL: *d_len)
  const int* d_len;
  double log2_rope_base;
  int* status;
  // split-K: grid z = splits CTAs per output tile, each over k blocks
  // [z*kb/splits, (z+1)*kb/splits); fp32 partial tiles part[(tile*splits+z)]
  // (128 x 256) and per-tile counters cnt[0..1024) (zero between launches):
  // the whole grid is resident, the CTAs of a tile wait for one another and
  // CTA z adds the partials in z order for its 1/splits of the epilogue
  // (RESID: its sums of squares go to ssq_out entry T * splits + z).
  int splits;
  float* part;
  int* cnt;
  // QKV: (cos, sin) of the RoPE angle of row tok and frequency j at
  // rope_cs[tok * 64 + j] (launch_rope_table fills it for these arguments)
  const float2* rope_cs;
  // QKV of the fused draft+verify forward (quad_B = B > 0): rows 0..B-1 are
  // the verify rows (slots L..L+B-1, K/V to the cache); row B + i*B + r is row
  // r of candidate block i at position L+i+1+r, its K/V to kside
  // [Hkv][side_n][128] / vside [Hkv][128][side_n] at key i*64 + r
  // (side_n >= 64 * B keys per KV head).
  int quad_B;
  bf16* kside;
  bf16* vside;
  int side_n;
};
// y = x W^T over n_wtiles tiles of 256 weight rows (SWIGLU: 128 rows of W and
// the same 128 rows of W2) starting at weight row w_row_base; kb = K / 64.
// (cos, sin) of every row's RoPE angles for the token-major QKV epilogue:
// row tok sits at position L0 + tok (L0 = *d_len when set), or for the
// candidate rows of a fused draft+verify forward (quad_B > 0, tok >= B) at
// L0 + i + 1 + r for row r of block i; frequency j of 64 is
// base^(-2j/128).  Angles and sincos in fp64, rounded to fp32.
cudaError_t launch_rope_table(float2* cs, const TmArgs& a, cudaStream_t s);
cudaError_t launch_gemm_tm(const CUtensorMap& mapX, const CUtensorMap& mapW, const CUtensorMap& mapW2, int kb,
                           int w_row_base, int n_wtiles, const TmArgs& a, cudaStream_t s);
struct PrefillAttnArgs {
  int n_tok, L0;              // query rows at slots L0..L0+n_tok-1
  int kv_base;                // cache entry (the layer)
  int Lmax, Hq, Hkv;
  float scale_log2;
  bf16* out;                  // [n_tok][out_ld], head h at column h * 128
  int out_ld;
  int* status;
};
cudaError_t launch_attn_prefill(const CUtensorMap& mapQ, const CUtensorMap& mapK, const CUtensorMap& mapV,
                                const PrefillAttnArgs& a, cudaStream_t s);

// FP8 E4M3 row quantisation (csrc/fp8.cu): codes [rows][K], scales [rows].
cudaError_t launch_quantize_rows_e4m3(const bf16* a, int rows, int K, uint8_t* codes, float* scales, cudaStream_t s);

// Embedding gather / row copy + per-128-feature sums of squares.
cudaError_t launch_embed_bf16(const bf16* E, const bf16* rows_in, int n_src, const int32_t* tokens,
                              const uint8_t* masked, int mask_id, int n_rows, int H, int V, bf16* x,
                              float* ssq_out, int NT, int* status, bool pdl, cudaStream_t s);

// Speculative accept.
cudaError_t launch_spec_logits(const bf16* logits, const int32_t* draft, int b, int B, int V, int32_t* accept_len,
                               int32_t* cache_len, int poison, bf16* kc, bf16* vc, int n_layers, int Hkv, int D,
                               int Lmax, float* ws_part, int* ws_cnt, int splits, int* status, cudaStream_t s);
cudaError_t launch_spec_ids(const int32_t* vids, const int32_t* draft, int b, int B, int32_t* accept_len,
                            int32_t* cache_len, int poison, bf16* kc, bf16* vc, int n_layers, int Hkv, int D,
                            int Lmax, int* status, cudaStream_t s);
// Decode-driver accept: k over (verify ids, draft), L = L - B + k, seed, emit.
cudaError_t launch_decode_accept(const int32_t* vids, const int32_t* draft, int B, int32_t* d_len,
                                 int32_t* seed, int32_t* out, int32_t* n_out, int max_new, int64_t* accept_hist,
                                 int32_t* k_out, int* status, bool pdl, cudaStream_t s);
// Fused draft+verify forward helpers: its input tokens, and the chosen
// candidate block's rows into the decode rows.
cudaError_t launch_quad_tokens(const int32_t* draft, int B, int mask_id, int32_t* qtok, cudaStream_t s);
cudaError_t launch_select_cand_rows(const bf16* src, int H, const int32_t* k_dev, int B, bf16* x, float* ssq_out,
                                    int NT, cudaStream_t s);
// Failure-detection self-test of the bounded waits.
cudaError_t launch_selftest_timeout(long long budget, int* status, int* waited_out, cudaStream_t s);
// Block bookkeeping for the decode driver.
cudaError_t launch_block_init(int32_t* tokens, uint8_t* masked, const int32_t* seed, int B, int mask_id,
                              int ar_seed, int32_t* n_remaining, cudaStream_t s);
cudaError_t launch_emit(const int32_t* tokens, int n, int32_t* out, int32_t* n_out, int max_new,
                        bool pdl, cudaStream_t s);

// fp32 CUDA-core path (tiny fp32 model).
cudaError_t f32_embed(const float* E, const float* rows_in, int n_src, const int32_t* tokens,
                      const uint8_t* masked, int mask_id, int n_rows, int H, int V, float* x, int* status,
                      cudaStream_t s);
cudaError_t f32_rowscale(const float* x, int ld, int n_rows, int H, float eps, float* r, cudaStream_t s);
cudaError_t f32_gemm(const float* x, int ld_x, const float* W, int n_out, int K, int n_rows, const float* r,
                     float* y, int ld_y, cudaStream_t s);
cudaError_t f32_rope_scatter(const float* y, int n_rows, int nq, int nkv, int D, const int* d_len, int L_static,
                             double log2_base, float* q_out, float* kc, float* vc, int Lmax, cudaStream_t s);
cudaError_t f32_add(float* resid, int ld_r, const float* y, int ld_y, int n_rows, int H, cudaStream_t s);
cudaError_t f32_swiglu(const float* g, const float* u, float* act, int n, cudaStream_t s);
cudaError_t f32_attention(const float* q, float* out, const float* kc, const float* vc, int n_batch, int n_rows,
                          int n_clean, int L, const int* d_len, int Lmax, int Hq, int Hkv, int D, float scale,
                          cudaStream_t s);
cudaError_t f32_lmhead(const float* hidden, const float* w, int R, int H, int V, const float* r, float* p1_buf,
                       int32_t* id_buf, const LmArgs& a, cudaStream_t s);

// Tensor maps (host).
bool make_tmap_2d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint64_t row_bytes,
                  uint32_t box_inner, uint32_t box_outer);
// Same for a byte matrix (E4M3 codes), 128-byte swizzle.
bool make_tmap_2d_u8(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint64_t row_bytes,
                     uint32_t box_inner, uint32_t box_outer);
bool make_tmap_3d(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t s1_bytes,
                  uint64_t s2_bytes, uint32_t b0, uint32_t b1, uint32_t b2);

}  // namespace dvlm
