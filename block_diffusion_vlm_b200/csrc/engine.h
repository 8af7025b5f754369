// Decode engine: owns host-side plans (tensor maps, CUDA graphs) over caller
// memory and drives the block-diffusion decode step.
#pragma once
#include <map>
#include <vector>

#include "kernels.h"

struct dvlm_engine;

namespace dvlm {

constexpr int kNT = 16;  // token rows per forward (block size <= 16)

// Per-kernel-class CUDA-event timing of one eager forward (profiling hook).
enum KernelKind { K_EMBED = 0, K_QKV, K_ATTN, K_OPROJ, K_GATEUP, K_DOWN, K_LMHEAD, K_CHAIN, K_KINDS };
struct KernelTimer {
  std::vector<std::pair<int, std::pair<cudaEvent_t, cudaEvent_t>>> marks;
  cudaStream_t s = nullptr;
  cudaEvent_t open = nullptr;
  void begin(int) {
    cudaEventCreate(&open);
    cudaEventRecord(open, s);
  }
  void end(int kind) {
    cudaEvent_t e;
    cudaEventCreate(&e);
    cudaEventRecord(e, s);
    marks.push_back({kind, {open, e}});
  }
};

// Where a forward's rows come from and what its LM head does.
struct FwdSpec {
  const void* rows_in = nullptr;  // first n_src rows copied from here
  int n_src = 0;
  const int32_t* tokens = nullptr;
  const uint8_t* masked = nullptr;
  int n_rows = 0;
  int n_clean = 0;
  int layer0 = 0;
  int n_layers = -1;         // -1: all
  bool advance = false;      // L += n_rows at the end
  bool lm = false;           // run the LM head
  LmArgs lma{};              // LM-head outputs (scratch pointers filled by the engine)
  void* x_out = nullptr;     // copy of the residual stream (test hook)
  KernelTimer* timer = nullptr;
  // TEXT-ONLY pass of certificate-guided routing: cache slots 0..hide-1 (the
  // vision rows) are hidden from attention, positions unchanged; L_host is
  // the cache length, read by the caller (eager forwards only).
  int hide = 0;
  int L_host = 0;
};

// Trace of the decode driver's forwards (test hook): one record per forward
// in a caller-owned device buffer, in launch order.  Layout of a record (32-bit
// words, then the final residual stream of its rows):
//   [0] kind (TR_*), [1] cache length L at the forward, [2] rows, [3] clean
//   rows, [4] LM-head rows R, [5..7] zero;
//   [8..23] block tokens before, [24..39] masked flags before (1 = masked),
//   [40..55] LM-head top-1 id of rows 0..R-1, [56..71] their top-1
//   probability (fp32 bits), [72..87] tokens after, [88..103] masked after,
//   [104] next AR seed after, [105] cache length after, [106..111] zero;
//   then rows x H residual-stream values (bf16 or fp32, the model's dtype),
//   before the final RMSNorm.  Records are padded to 256 bytes.
enum TraceKind { TR_NOISY = 1, TR_APPEND = 2, TR_DRAFT = 3, TR_VERIFY = 4, TR_AR = 5, TR_QUAD_VERIFY = 6,
                 TR_QUAD_CAND = 7, TR_ROUTE_FULL = 8, TR_ROUTE_TEXT = 9 };
constexpr int kQuadSideKeys = 16 * 64;
constexpr int kMaxAttnSplit = 32;  // side-buffer keys per head: candidate block i at i * 64
constexpr int kTraceWords = 112;
inline size_t trace_record_bytes(int hidden, bool bf16) {
  const size_t b = kTraceWords * 4 + static_cast<size_t>(kNT) * hidden * (bf16 ? 2 : 4);
  return (b + 255) / 256 * 256;
}

// Kernel launches of one forward pass over n_layers layers.
inline int launches_per_forward(int n_layers) { return 2 + 5 * n_layers; }

}  // namespace dvlm

struct dvlm_engine {
  dvlm_model m{};
  bool bf16 = true;
  bool fp8 = false;                     // FP8 W8A8 projections (bf16 everywhere else)
  int Lmax = 0, max_block = 0, max_ctx = 0;
  void* kc = nullptr;
  void* vc = nullptr;
  int sm = 0;
  int s_qkv = 0, s_o = 0, s_down = 0;  // cluster sizes of the split-K projections (0: stream-K)
  int attn_cs = 8;                      // CTAs per attention cluster (8 or 16)
  int attn_split = 0;                   // > 0: split attention with this many CTAs per KV head
  int gu_stages = 10, down_stages = 10; // pipeline depth of the gate/up and down projections
  int gu_cps = 1;                       // gate/up CTAs per SM (2 needs 5 stages)
  bool pdl = true;                      // programmatic dependent launch between kernels
  bool prefill_gemm = true;             // compute-bound prefill (prefill.cu) where the shapes allow it
  // paged KV cache (dvlm_engine_set_paged): kc / vc are 64-slot pages
  // [n_layers][n_pages][Hkv][64][D] and [n_layers][n_pages][Hkv][D][64]
  bool paged = false;
  const int32_t* block_table = nullptr;  // [max_pages] page of each 64-slot chunk
  int n_pages = 0, max_pages = 0;
  // device buffers carved from the workspace
  void* x = nullptr;        // [NT][H]
  void* q = nullptr;        // [NT][Hq*D]
  void* attn_o = nullptr;   // [NT][Hq*D]
  void* act = nullptr;      // [NT][I]
  float* ssq = nullptr;     // [H/128][NT]
  float* gpart = nullptr;   // GEMM split scratch
  int* gcnt = nullptr;      // split-tile counters, one block of gcnt_stride per chain phase
  int gcnt_stride = 0;
  int* chain_bar = nullptr; // persistent forward: barrier and exit counters
  void* fwd_att = nullptr;  // persistent forward: attention partials and (max, sum) per 64-key chunk
  bool chain = false;       // the whole forward as one persistent launch (option "persistent")
  float* lpart = nullptr;   // LM head scratch
  int* lcnt = nullptr;
  float* lrec = nullptr;
  int* ldone = nullptr;
  int32_t* d_len = nullptr;
  int32_t* d_seed = nullptr;
  int* d_status = nullptr;
  int32_t* tokens = nullptr;     // [NT+1]
  uint8_t* masked = nullptr;     // [NT+1]
  int32_t* n_remaining = nullptr;
  int32_t* vids = nullptr;       // [NT+1]
  int32_t* n_out = nullptr;
  int64_t* hist = nullptr;       // commit histogram [DVLM_HIST]
  int64_t* ahist = nullptr;      // accept histogram [DVLM_HIST]
  void* stage_vis = nullptr;     // [max_ctx][H]
  int32_t* stage_ids = nullptr;  // [max_ctx]
  int32_t* stage_out = nullptr;  // [max_ctx] generated tokens (host path)
  int32_t* h_pinned = nullptr;   // host-mapped scalars (n_remaining, n_out, L, seed)
  // certificate-guided routing: anchors (FULL pass), TEXT-ONLY outputs, certified length
  int32_t* anc_id = nullptr;     // [NT]
  float* anc_p1 = nullptr;       // [NT]
  int32_t* txt_id = nullptr;     // [NT]
  float* txt_p1 = nullptr;       // [NT]
  int32_t* cert = nullptr;       // [1]
  int32_t* tr_top1 = nullptr;    // [NT] LM-head ids while tracing
  float* tr_p1 = nullptr;        // [NT] LM-head probabilities while tracing
  // forward trace (test hook, off unless set): records, capacity, device count
  uint8_t* trace_buf = nullptr;
  int trace_cap = 0;
  int32_t* trace_cnt = nullptr;
  // compute-bound prefill buffers, max_ctx rows each (bf16 engines)
  void* px = nullptr;            // [max_ctx][H] residual stream
  void* pq = nullptr;            // [max_ctx][Hq*D]
  void* pao = nullptr;           // [max_ctx][Hq*D] attention output
  void* pact = nullptr;          // [max_ctx][I] SwiGLU activation
  float* pssq = nullptr;         // [max(H/128 + 1, 16 H/256)][max_ctx] sums of squares
  float2* rope_cs = nullptr;     // [max_ctx][64] (cos, sin) of each context row's RoPE angles
  float* amax_act = nullptr;     // fp8: [I/64][NT] largest |SwiGLU activation| per gate/up tile
  void* attn_scratch = nullptr;  // split attention partials (up to kMaxAttnSplit CTAs per KV head)
  // quadratic self-speculative decoding (fused draft + verify forward)
  int32_t* qtok = nullptr;       // [max_ctx] input tokens of the fused forward
  int32_t* d_k = nullptr;        // accepted length of the last fused round
  void* kside = nullptr;         // candidate K [Hkv][16*64][128] (one layer at a time)
  void* vside = nullptr;         // candidate V^T [Hkv][128][16*64]
  float* qpart = nullptr;        // split-K partial tiles of the token-major GEMMs
  int* qcnt = nullptr;           // their per-tile counters (zero between launches)
  bool quad_ready = false;       // the next fused round's draft is in `tokens`
  int quad_B = 0;
  // fp32 path scratch
  float* f_y = nullptr;          // [NT][max(qkv_rows, H)]
  float* f_r = nullptr;          // [NT]
  float* f_g = nullptr;          // [NT][I]
  float* f_u = nullptr;          // [NT][I]
  float* f_p1 = nullptr;         // [NT]
  int32_t* f_id = nullptr;       // [NT]
  // tensor maps
  CUtensorMap tm_wqkv, tm_wo, tm_wg, tm_wu, tm_wd, tm_lm, tm_x, tm_ao, tm_act, tm_q, tm_k, tm_v;
  // prefill: activations (128-row boxes), weights (256-row boxes; gate/up 128), K (128-key boxes)
  CUtensorMap tm_px, tm_pq, tm_pao, tm_pact, tm_wqkv_p, tm_wo_p, tm_wd_p, tm_wg_p, tm_wu_p, tm_kp;
  // fused forward: q rows as 16-row x 8-head boxes, candidate side buffers
  CUtensorMap tm_q3, tm_ks, tm_vs;  // quad: q rows (3-D), side K and V^T with the decode attention's boxes
  // captured graphs keyed by (kind, B, threshold bits, max_new)
  std::map<std::vector<long long>, cudaGraphExec_t> graphs;
};
