// Commit / certificate / bookkeeping over the rows of one LM-head call, run by
// 128 threads (one row each, R <= 128) once every row's top-1 probability and
// id are known.  Shared by the tensor-core LM head and the fp32 path.
//   commit:      masked rows with p1 >= threshold; if none, the masked row
//                with the highest p1 (lowest row on ties)
//                [Fast-dVLM technical overview (ocdem.com), section 4.1:
//                threshold 0.9; at least one position per step];
//   certificate: rows masked on entry, visited by descending anchor
//                confidence (lower row first on ties); count until the
//                first row whose id differs from its anchor
//                [Look Only When Needed, method step (2)].
#pragma once
#include "kernels.h"

namespace dvlm {

struct FinalizeSmem {
  float p1[128];
  float conf[128];
  int id[128];
  int msk[128];
  int npass, best, ncommit, nmasked, cert;
};

template <typename Bar>
__device__ void finalize_rows(int tid, const LmArgs& a, FinalizeSmem& fs, Bar bar) {
  const int R = a.R;
  const int r = tid;
  const bool valid = r < R;
  const float p = valid ? fs.p1[r] : -1.0f;
  const int id = valid ? fs.id[r] : 0;
  const bool msk = valid && (a.masked ? (a.masked[r] != 0) : true);
  const bool have_cert = a.anchor_id && a.anchor_conf && a.cert_len;
  fs.msk[r] = msk ? 1 : 0;
  if (have_cert) fs.conf[r] = valid ? a.anchor_conf[r] : 0.0f;
  if (tid == 0) {
    fs.npass = 0;
    fs.best = -1;
    fs.ncommit = 0;
    fs.nmasked = 0;
    fs.cert = 0;
  }
  bar();
  const bool pass = msk && p >= a.threshold;
  if (pass) atomicAdd(&fs.npass, 1);
  if (msk) atomicAdd(&fs.nmasked, 1);
  bar();
  if (tid == 0 && fs.npass == 0) {
    int best = -1;
    for (int j = 0; j < R; ++j)
      if (fs.msk[j] && (best < 0 || fs.p1[j] > fs.p1[best])) best = j;
    fs.best = best;
  }
  if (have_cert && tid == 0) fs.cert = fs.nmasked;
  bar();
  const bool com = pass || (fs.npass == 0 && r == fs.best);
  if (valid) {
    if (a.top1_id) a.top1_id[r] = id;
    if (a.top1_prob) a.top1_prob[r] = p;
    if (a.commit) a.commit[r] = com ? 1 : 0;
    if (a.id_out) a.id_out[r] = id;
    if (com && a.tokens) {
      a.tokens[r] = id;
      a.masked[r] = 0;
    }
    if (a.seed_out && r == a.seed_row) *a.seed_out = id;
  }
  if (com) atomicAdd(&fs.ncommit, 1);
  if (have_cert && msk && id != a.anchor_id[r]) {
    const float c = fs.conf[r];
    int rank = 0;
    for (int j = 0; j < R; ++j)
      if (fs.msk[j] && (fs.conf[j] > c || (fs.conf[j] == c && j < r))) ++rank;
    atomicMin(&fs.cert, rank);
  }
  bar();
  if (tid == 0) {
    if (a.n_commit) *a.n_commit = fs.ncommit;
    if (a.n_remaining) *a.n_remaining = fs.nmasked - (a.tokens ? fs.ncommit : 0);
    if (a.hist && fs.ncommit < DVLM_HIST) atomicAdd(reinterpret_cast<unsigned long long*>(&a.hist[fs.ncommit]), 1ull);
    if (a.nfe) atomicAdd(reinterpret_cast<unsigned long long*>(a.nfe), 1ull);
    if (have_cert) *a.cert_len = fs.cert;
    if (a.len_ptr) *a.len_ptr += a.len_advance;
  }
  bar();
}

}  // namespace dvlm
