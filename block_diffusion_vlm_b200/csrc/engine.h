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
enum KernelKind { K_EMBED = 0, K_QKV, K_ATTN, K_OPROJ, K_GATEUP, K_DOWN, K_LMHEAD, K_KINDS };
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

// Kernel launches of one forward pass over n_layers layers.
inline int launches_per_forward(int n_layers) { return 2 + 5 * n_layers; }

}  // namespace dvlm

struct dvlm_engine {
  dvlm_model m{};
  bool bf16 = true;
  int Lmax = 0, max_block = 0, max_ctx = 0;
  void* kc = nullptr;
  void* vc = nullptr;
  int sm = 0;
  int s_qkv = 0, s_o = 0, s_down = 0;  // cluster sizes of the split-K projections (0: stream-K)
  int attn_cs = 8;                      // CTAs per attention cluster (8 or 16)
  int gu_stages = 10, down_stages = 10; // pipeline depth of the gate/up and down projections
  int gu_cps = 1;                       // gate/up CTAs per SM (2 needs 5 stages)
  bool pdl = true;                      // programmatic dependent launch between kernels
  // device buffers carved from the workspace
  void* x = nullptr;        // [NT][H]
  void* q = nullptr;        // [NT][Hq*D]
  void* attn_o = nullptr;   // [NT][Hq*D]
  void* act = nullptr;      // [NT][I]
  float* ssq = nullptr;     // [H/128][NT]
  float* gpart = nullptr;   // GEMM split scratch
  int* gcnt = nullptr;
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
  // fp32 path scratch
  float* f_y = nullptr;          // [NT][max(qkv_rows, H)]
  float* f_r = nullptr;          // [NT]
  float* f_g = nullptr;          // [NT][I]
  float* f_u = nullptr;          // [NT][I]
  float* f_p1 = nullptr;         // [NT]
  int32_t* f_id = nullptr;       // [NT]
  // tensor maps
  CUtensorMap tm_wqkv, tm_wo, tm_wg, tm_wu, tm_wd, tm_lm, tm_x, tm_ao, tm_act, tm_q, tm_k, tm_v;
  // captured graphs keyed by (kind, B, threshold bits, max_new)
  std::map<std::vector<long long>, cudaGraphExec_t> graphs;
};
