// Block-masked GQA attention against the exact KV cache, bf16, tcgen05.
//
// Visibility [Fast-dVLM technical overview (ocdem.com), section 2.2.1;
// Fast-dVLM walkthrough (itsolotime.com), section 4.1]: a clean row t (slot
// L+t) sees slots 0..L+t (C2C, causal); a noisy row sees every slot
// 0..L+n_rows-1 -- the whole cache of vision, prompt and committed tokens
// (N2C) and its own block in both directions (N2N).
//
// Tile: one KV head's 8 query heads x 16 step rows = 128 rows (token-major,
// head-minor, as a 3-D TMA box lands).  Keys go in 128-key chunks, chunk j
// to split j % S (round robin by absolute key position, so a causal row's
// arithmetic is the same whatever the number of rows in the step: a 1-row AR
// pass and a 16-row verify pass give bitwise the same output).  Each of the S
// CTAs of a (batch entry, row group, KV head) streams its chunks through
// two key and two value stages (TMA); S = Q K^T and O += P V accumulate in
// TMEM with Q and P as TMEM operands; the online softmax runs in fp32 with
// two threads per row, one per 64-key half, P in fp16 (the value tile
// converted to fp16 in shared memory by two dedicated warps); the running
// maximum moves only when a score passes it by more than 2^8, which leaves
// the result exact up to rounding and skips most rescales of O.
//
// Two ways to merge the S partials (O / l and (m, l) per row):
//   split form (kCL = 0, the bandwidth-bound form): fp32 partial rows to
//   global scratch, a counter per group, the last CTA to arrive merges in
//   split order; no CTA waits for another;
//   cluster form (kCL = S = 8 or 16, the decode path and the candidate blocks
//   of the quadratic forward): the S CTAs are one thread-block cluster; fp16
//   partial rows go by bulk copies straight into the shared memory of the
//   CTA owning those rows, which merges them in source order; no scratch, no
//   second kernel.
// Paged caches read each 64-key half chunk through the block table.
#include <cuda_fp16.h>

#include "kernels.h"
#include "mainloop.cuh"

namespace dvlm {

namespace {
constexpr int kSpThreads = 384;        // warp 0 TMA, 1 MMA, 2..9 softmax (two per TMEM lane quarter), 10..11 value conversion
constexpr int kSpSoftmax = 256;        // softmax threads: row = quarter * 32 + lane, key half = (warp - 2) / 4
constexpr float kSpLazy = 8.0f;        // log2 headroom before the running maximum moves
constexpr int kSpPrefetch = 4;         // L2 prefetch distance in chunks past the newest load
constexpr int kSpKeys = 128;           // keys per chunk
constexpr int kSpAtom = 128 * 128;     // one 128-byte-swizzled 128-row operand atom (16 KB)
constexpr int oSpQ = 0;                // Q: 2 atoms (d 0..63, 64..127)
constexpr int kSpStages = 2;           // key stages and value stages (each)
constexpr int oSpK = oSpQ + 2 * kSpAtom;   // K: kSpStages x 2 d-atoms
constexpr int oSpV = oSpK + 2 * kSpStages * kSpAtom;   // V^T: kSpStages x 2 key-atoms
constexpr int oSpBar = oSpV + 2 * kSpStages * kSpAtom;
constexpr int oSpL = oSpBar + 256;     // [2][128] row sums of the two key halves
constexpr int oSpMx = oSpL + 1024;     // [2 chunk parities][2 halves][128] half-chunk row maxima
constexpr int oSpRecv = oSpMx + 2048;  // cluster merge: [source CTA][row of this CTA][128] fp16 O / l
constexpr int oSpRecvML = oSpRecv + 128 * 128 * 2;  // and [source CTA][row] (m, l)
constexpr int kSpSmem = oSpRecvML + 128 * 8 + 1024;
constexpr uint32_t kSpIdescS = idesc_bf16_f32(128, kSpKeys);
constexpr uint32_t kSpIdescO = idesc_f16_f32(128, 128);
constexpr int kSpTmem = 512;
// TMEM columns: S of the two buffers, O (fp32), and the two operands the
// products take from TMEM instead of shared memory: P (fp16, two keys per
// column) and Q (bf16, two features per column, staged once per CTA)
constexpr uint32_t kSpColO = 256, kSpColP = 384, kSpColQ = 448;
}  // namespace

size_t attn_split_scratch_bytes(int n_groups_total, int S) {
  const size_t part = static_cast<size_t>(n_groups_total) * S * 128 * 128 * 4;
  const size_t ml = static_cast<size_t>(n_groups_total) * S * 128 * 8;
  return (part + 255) / 256 * 256 + (ml + 255) / 256 * 256 + (static_cast<size_t>(n_groups_total) * 4 + 255) / 256 * 256;
}

// kCL = 0: S = gridDim.x independent CTAs, partials through global scratch,
// merged by the last CTA of the group.  kCL = 8 or 16: the S = kCL CTAs of a
// group form one thread-block cluster; each CTA with keys bulk-copies its
// fp16 partial rows O / l and (m, l) straight into the shared memory of the
// CTA that owns those rows (128 / kCL rows each), counted on that CTA's
// receive barrier, and the owner merges them: no global scratch, no counter.
// Candidate blocks of a fused draft+verify forward (a.cand_B > 0, cluster
// form) are batch entries whose key set is a cache prefix plus one side
// chunk of the block's own keys (AttnArgs).
template <int kCL>
__global__ void __launch_bounds__(kSpThreads, 1)
    attn_split_kernel(const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapK,
                      const __grid_constant__ CUtensorMap mapV, const __grid_constant__ CUtensorMap mapKs,
                      const __grid_constant__ CUtensorMap mapVs, const AttnArgs a, float* part, float2* ml,
                      int* cnt) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sQ = smem + oSpQ;
  uint8_t* sK = smem + oSpK;
  uint8_t* sV = smem + oSpV;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + oSpBar);
  uint64_t* q_full = bars;
  uint64_t* s_full = bars + 1;    // [2]
  uint64_t* s_empty = bars + 3;   // [2] the softmax warps have read S of that buffer
  uint64_t* p_full = bars + 5;    // P of the current chunk written, O rescaled (one phase per chunk)
  uint64_t* pv_done = bars + 6;   // PV of a chunk done (one phase per chunk)
  uint64_t* q_tmem = bars + 7;    // Q staged into TMEM by the softmax warps
  uint64_t* k_full = bars + 8;                   // [kSpStages] keys of the chunk in that stage landed
  uint64_t* k_empty = k_full + kSpStages;        // [kSpStages] S of that chunk done (its keys are free)
  uint64_t* v_full = k_empty + kSpStages;        // [kSpStages] values of the chunk in that stage landed
  uint64_t* v_empty = v_full + kSpStages;        // [kSpStages] PV of that chunk done (its values are free)
  uint64_t* v_conv = v_empty + kSpStages;        // [kSpStages] values of that chunk converted to fp16
  uint64_t* mx_bar = v_conv + kSpStages;         // [4 quarters][2 chunk parities] both halves' maxima written
  uint64_t* recv_full = mx_bar + 8;              // cluster merge: every sending CTA's rows landed
  constexpr int kSpBars = 8 + 5 * kSpStages + 8 + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kSpBars);
  volatile int* sabort = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* sflag = reinterpret_cast<int*>(tmem_slot + 2);
  float* sLh = reinterpret_cast<float*>(smem + oSpL);
  float* sMx = reinterpret_cast<float*>(smem + oSpMx);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = gridDim.x, sp = blockIdx.x, g = blockIdx.y;
  const int n_groups = (a.n_rows + 15) / 16;
  const int bidx = blockIdx.z / n_groups;
  const int t_base = (blockIdx.z % n_groups) * 16;
  const int grp = blockIdx.z * a.Hkv + g;  // one merge group per (batch entry, row group, KV head)

  // The cache length is final before this kernel's predecessor runs (only the
  // end of a forward pass moves it), and so are the slots below it: both are
  // read before waiting for the predecessor.  Slots L.. and the queries come
  // from the QKV projection this kernel follows: the loader waits for it
  // before those loads, and every other input of the kernel reaches it
  // through the loader's copies.
  // candidate block bidx (cand_B > 0): the cache prefix 0..*d_len + bidx,
  // then one side chunk of its own cand_B keys
  const bool cand = a.cand_B > 0;
  const int L_old = a.d_len ? *a.d_len : a.L_static;  // slots below it predate the predecessor
  int L = cand ? L_old + bidx + 1 : (a.d_lens ? a.d_lens[bidx] : L_old) - a.len_sub;
  if (a.block_table && L + a.n_rows > a.max_pages * 64) {
    record_error(a.status, DVLM_ERR_BOUNDS);
    L = a.max_pages * 64 - a.n_rows;
  }
  const int Ltot = cand ? L : L + a.n_rows;  // cache slots this entry's rows may see
  const int n_cache = (Ltot + kSpKeys - 1) / kSpKeys;
  const int n_all = n_cache + (cand ? 1 : 0);
  const int nc = sp < n_all ? (n_all - sp + S - 1) / S : 0;  // this CTA's chunks sp, sp+S, ...
  // (cache entry, KV head) row block: batch entry b reads cache entry kv_base + b; the candidate
  // blocks all read entry kv_base
  const int kv_row0 = (a.kv_base + (cand ? 0 : bidx)) * a.Hkv + g;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kSpBars; ++i) {
      const bool pair = &bars[i] >= v_conv && &bars[i] < recv_full;  // v_conv, mx_bar: two arrivals
      mbar_init(&bars[i], (i >= 3 && i <= 5) || i == 7 ? 8 : (pair ? 2 : 1));
    }
    if constexpr (kCL > 0)  // the CTAs with keys send RPC rows of fp16 O / l and of (m, l) each
      mbar_arrive_expect_tx(recv_full, static_cast<uint32_t>(min(kCL, n_all)) * (128 / kCL) * (256 + 8));
    *sabort = 0;
    fence_mbar_init();
    tma_prefetch_map(&mapQ);
    tma_prefetch_map(&mapK);
    tma_prefetch_map(&mapV);
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, kSpTmem);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // every CTA of the cluster is running before any sends into it (the wait
  // sits just before the sends)
  if constexpr (kCL > 0) cluster_arrive();

  // (layer, page, head) entry holding logical slot `key` of a paged cache
  auto page_entry = [&](int key) -> int {
    int page = a.block_table[bidx * a.max_pages + key / 64];
    if (page < 0 || page >= a.n_pages) {
      record_error(a.status, DVLM_ERR_BOUNDS);
      page = 0;
    }
    return (a.kv_base * a.n_pages + page) * a.Hkv + g;
  };

  if (warp == 0) {
    if (lane == 0 && nc > 0) {
      const uint64_t pol = l2_policy_evict_first();
      // coordinates of 64-key half `hf` of this CTA's chunk c (one page each
      // in a paged cache)
      // (the side chunk of a candidate block: rows of the side buffers; a
      // half past its 64 keys reads the next block's rows or zero fill)
      auto coords = [&](int c, int hf, int& krow, int& vrow, int& vx) -> bool {
        const int key = (sp + c * S) * kSpKeys + hf * 64;
        if (cand && sp + c * S == n_cache) {
          krow = g * a.side_n + bidx * 64 + hf * 64;
          vrow = g * 128;
          vx = bidx * 64 + hf * 64;
          return true;
        }
        if (a.block_table) {
          const int pe = page_entry(key);
          krow = pe * 64;
          vrow = pe * 128;
          vx = 0;
        } else {
          krow = kv_row0 * a.Lmax + key;
          vrow = kv_row0 * 128;
          vx = key;
        }
        return false;
      };
      // Keys and values have two stages each, released separately: a key
      // stage as soon as S of its chunk is done, a value stage once PV is.
      // Keys therefore run one chunk ahead of values (K(i) is issued before
      // V(i - 1), the order in which their stages free up).  The chunks after
      // the loaded ones are prefetched into L2 (up to kSpPrefetch ahead of the
      // newest key load), so a refill reads L2 instead of DRAM.
      auto load_k = [&](int c) {
        const int st = c % kSpStages;
        mbar_arrive_expect_tx(&k_full[st], 2 * kSpAtom);
        for (int hf = 0; hf < 2; ++hf) {
          int krow, vrow, vx;
          const CUtensorMap* mk = coords(c, hf, krow, vrow, vx) ? &mapKs : &mapK;
          for (int d = 0; d < 2; ++d)
            tma_load_2d(sK + (2 * st + d) * kSpAtom + hf * (kSpAtom / 2), mk, &k_full[st], d * 64, krow, pol);
        }
      };
      auto load_v = [&](int c) {
        const int st = c % kSpStages;
        mbar_arrive_expect_tx(&v_full[st], 2 * kSpAtom);
        for (int hf = 0; hf < 2; ++hf) {
          int krow, vrow, vx;
          const CUtensorMap* mv = coords(c, hf, krow, vrow, vx) ? &mapVs : &mapV;
          tma_load_2d(sV + (2 * st + hf) * kSpAtom, mv, &v_full[st], vx, vrow, pol);
        }
      };
      // the first stages' chunks that lie wholly below the cache length load
      // before the wait for the predecessor
      bool early[kSpStages];
      for (int c = 0; c < kSpStages; ++c) {
        early[c] = c < nc && (sp + c * S + 1) * kSpKeys <= (cand ? L_old : L);
        if (early[c]) {
          load_k(c);
          load_v(c);
        }
      }
      griddep_wait();
      mbar_arrive_expect_tx(q_full, 2 * kSpAtom);
      for (int d = 0; d < 2; ++d)
        tma_load_3d(sQ + d * kSpAtom, &mapQ, q_full, d * 64, g * 8, a.q_row0 + bidx * a.n_rows + t_base, pol);
      int pf = kSpStages;
      for (int i = 0; i <= nc; ++i) {
        if (i < nc) {
          if (i >= kSpStages && !mbar_wait(&k_empty[i % kSpStages], ((i / kSpStages) - 1) & 1, a.status, sabort))
            break;
          if (i >= kSpStages || !early[i]) load_k(i);
          for (; pf < nc && pf <= i + kSpPrefetch; ++pf) {
            for (int hf = 0; hf < 2; ++hf) {
              int krow, vrow, vx;
              const bool sd = coords(pf, hf, krow, vrow, vx);
              for (int d = 0; d < 2; ++d) tma_prefetch_2d(sd ? &mapKs : &mapK, d * 64, krow);
              tma_prefetch_2d(sd ? &mapVs : &mapV, vx, vrow);
            }
          }
        }
        if (i >= 1) {
          const int c = i - 1;
          if (c >= kSpStages && !mbar_wait(&v_empty[c % kSpStages], ((c / kSpStages) - 1) & 1, a.status, sabort))
            break;
          if (c >= kSpStages || !early[c]) load_v(c);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && nc > 0) {
      bool ok = mbar_wait(q_tmem, 0, a.status, sabort);
      // descriptors of stage 0's K and V tiles; a stage or K-step offset adds
      // (bytes >> 4) to the start-address field (addresses stay below 2^18)
      const uint64_t kdesc0 = sdesc_kmajor_sw128(smem_u32(sK)), vdesc0 = sdesc_kmajor_sw128(smem_u32(sV));
      auto issue_pv = [&](int c) -> bool {
        if (!mbar_wait(p_full, c & 1, a.status, sabort)) return false;
        tc_fence_after();
        const uint64_t vd = vdesc0 + static_cast<uint64_t>((2 * (c % kSpStages) * kSpAtom) >> 4);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          umma_f16_ts(tmem + kSpColO, tmem + kSpColP + kk * 8, vd + (((kk >> 2) * kSpAtom + (kk & 3) * 32) >> 4),
                      kSpIdescO, (c > 0 || kk > 0) ? 1u : 0u);
        umma_commit(&v_empty[c % kSpStages]);
        umma_commit(pv_done);
        return true;
      };
      // Issue whichever product is ready: PV of the oldest chunk with its P
      // written (that frees its K/V stage for the load two chunks ahead), else
      // S of the next chunk with its keys landed and its S buffer free.  A
      // fixed S(c), PV(c-1) order would hold every load back until the
      // previous one landed.
      int cs = 0, cp = 0;
      long long t0 = clock64();
      while (ok && cp < nc) {
        if (cp < cs && mbar_test_wait(p_full, cp & 1) &&
            mbar_test_wait(&v_conv[cp % kSpStages], (cp / kSpStages) & 1)) {
          ok = issue_pv(cp);
          ++cp;
          t0 = clock64();
          continue;
        }
        if (cs < nc && cs <= cp + 1) {
          const int st = cs & 1, ks = cs % kSpStages;
          if (mbar_test_wait(&k_full[ks], (cs / kSpStages) & 1) &&
              (cs < 2 || mbar_test_wait(&s_empty[st], ((cs >> 1) - 1) & 1))) {
            tc_fence_after();
            const uint64_t kd = kdesc0 + static_cast<uint64_t>((2 * ks * kSpAtom) >> 4);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              umma_f16_ts(tmem + st * kSpKeys, tmem + kSpColQ + kk * 8,
                          kd + (((kk >> 2) * kSpAtom + (kk & 3) * 32) >> 4), kSpIdescS, kk > 0 ? 1u : 0u);
            umma_commit(&k_empty[ks]);
            umma_commit(&s_full[st]);
            ++cs;
            t0 = clock64();
            continue;
          }
        }
        if (*sabort || clock64() - t0 > kWaitBudgetCycles) {
          record_error(a.status, DVLM_ERR_TIMEOUT);
          *sabort = 1;
          ok = false;
        }
      }
    }
  } else if (warp >= 10) {
    // ------------------------------------------------------ value conversion
    // Warp 10 + cw turns value rows (features) 64 cw .. 64 cw + 63 of each
    // chunk's two key atoms from bf16 to fp16 in place, two rows per lane;
    // keys past the valid slots (stale, poisoned, other pages' rows) become
    // 0.  All eight 16-byte pieces of a row are loaded first, then converted,
    // then stored.
    const int cw = warp - 10;
    for (int c = 0; c < nc; ++c) {
      const int vs = c % kSpStages;
      if (!mbar_wait(&v_full[vs], (c / kSpStages) & 1, a.status, sabort)) break;
      const bool side = cand && sp + c * S == n_cache;  // a candidate block's own keys
      const int key0 = side ? 0 : (sp + c * S) * kSpKeys;
#pragma unroll 1
      for (int j = 0; j < 4; ++j) {
        const int at = j & 1, d = 64 * cw + 32 * (j >> 1) + lane;
        const int n_valid = (side ? a.cand_B : Ltot) - key0 - at * 64;
        uint8_t* vrow = sV + (2 * vs + at) * kSpAtom + d * 128;
        uint4 w[8];
#pragma unroll
        for (int cc = 0; cc < 8; ++cc) w[cc] = *reinterpret_cast<const uint4*>(vrow + ((cc ^ (d & 7)) << 4));
        if (n_valid >= 64) {
#pragma unroll
          for (int cc = 0; cc < 8; ++cc) {
            uint32_t* wv = reinterpret_cast<uint32_t*>(&w[cc]);
#pragma unroll
            for (int e = 0; e < 4; ++e) wv[e] = bf16x2_to_f16x2(wv[e]);
          }
        } else {
#pragma unroll
          for (int cc = 0; cc < 8; ++cc) {
            uint32_t* wv = reinterpret_cast<uint32_t*>(&w[cc]);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int kk = (cc << 3) + 2 * e;
              const uint32_t keep = (kk < n_valid ? 0x0000FFFFu : 0u) | (kk + 1 < n_valid ? 0xFFFF0000u : 0u);
              wv[e] = bf16x2_to_f16x2(wv[e] & keep);
            }
          }
        }
#pragma unroll
        for (int cc = 0; cc < 8; ++cc) *reinterpret_cast<uint4*>(vrow + ((cc ^ (d & 7)) << 4)) = w[cc];
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&v_conv[vs]);
    }
  } else {
    // ---------------------------------------------------------------- softmax
    // Two warps per TMEM lane quarter: warp half `hf` exponentiates keys
    // 64 hf .. 64 hf + 63 of each chunk (P atom hf), rescales output features
    // 64 hf .. 64 hf + 63 and converts value atom hf.  Both warps of a quarter
    // take the row maximum over all 128 keys, so they hold the same (m, alpha)
    // without exchanging it; each keeps the row sum of its own keys.
    // The next kernel (the output projection) may launch now and stream its
    // weights on idle SMs; it reads this kernel's output only after its own
    // wait (at most two kernels overlap).
    if (threadIdx.x == 64) griddep_launch_dependents();
    const int quarter = warp & 3;
    const int hf = (warp - 2) >> 2;
    const int row = quarter * 32 + lane;
    const int t = t_base + (row >> 3);
    const int limit = (t < a.n_clean) ? (L + t + 1) : Ltot;  // keys below `limit` are visible
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    float m = -INFINITY, l = 0.f;
    bool ok = nc > 0;
    if (ok) {
      // Q row `row`, features 64 hf .. 64 hf + 63 (atom hf), into TMEM
      // columns kSpColQ + 32 hf .. + 31 for the S products
      ok = mbar_wait(q_full, 0, a.status, sabort);
      if (ok) {
        const uint8_t* qrow = sQ + hf * kSpAtom + row * 128;
        uint32_t qw[32];
#pragma unroll
        for (int cc = 0; cc < 8; ++cc) {
          const uint4 v = *reinterpret_cast<const uint4*>(qrow + ((cc ^ (row & 7)) << 4));
          qw[4 * cc] = v.x;
          qw[4 * cc + 1] = v.y;
          qw[4 * cc + 2] = v.z;
          qw[4 * cc + 3] = v.w;
        }
        tmem_st16u_nowait(tmem + lane_off + kSpColQ + hf * 32, qw);
        tmem_st16u_nowait(tmem + lane_off + kSpColQ + hf * 32 + 16, qw + 16);
        tmem_wait_st();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(q_tmem);
    }
    for (int c = 0; ok && c < nc; ++c) {
      const int st = c & 1;
      // chunk keys key0 .. key0 + 127 against the visible bound lim (the side
      // chunk of a candidate block: its own keys 0 .. cand_B - 1)
      const bool side = cand && sp + c * S == n_cache;
      const int key0 = side ? 0 : (sp + c * S) * kSpKeys;
      const int lim = side ? a.cand_B : limit;
      const bool full = key0 + kSpKeys <= lim;  // every key of the chunk visible to this row
      if (!mbar_wait(&s_full[st], (c >> 1) & 1, a.status, sabort)) {
        ok = false;
        break;
      }
      tc_fence_after();
      float sc[64];  // this warp's 64 keys
      tmem_ld64(tmem + lane_off + static_cast<uint32_t>(st * kSpKeys + hf * 64), sc);
      // maximum over this half (eight independent chains), then over the
      // row's two halves through shared memory (max is exact in any order,
      // so both warps hold the same value)
      float mv[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) mv[j] = -INFINITY;
      if (full) {
#pragma unroll
        for (int k = 0; k < 64; ++k) mv[k & 7] = fmaxf(mv[k & 7], sc[k]);
      } else {
        const int kme = key0 + hf * 64;
#pragma unroll
        for (int k = 0; k < 64; ++k)
          if (kme + k < lim) mv[k & 7] = fmaxf(mv[k & 7], sc[k]);
      }
      const float mh = fmaxf(fmaxf(fmaxf(mv[0], mv[1]), fmaxf(mv[2], mv[3])),
                             fmaxf(fmaxf(mv[4], mv[5]), fmaxf(mv[6], mv[7])));
      sMx[((c & 1) * 2 + hf) * 128 + row] = mh;
      __syncwarp();
      if (lane == 0) mbar_arrive(&mx_bar[quarter * 2 + (c & 1)]);
      if (!mbar_wait(&mx_bar[quarter * 2 + (c & 1)], (c >> 1) & 1, a.status, sabort)) {
        ok = false;
        break;
      }
      const float mx = fmaxf(mh, sMx[((c & 1) * 2 + (hf ^ 1)) * 128 + row]);
      // scale_log2 > 0, so the maximum of the scaled scores is the scaled
      // maximum (rounding is monotonic).  The reference maximum moves only
      // when a score exceeds it by more than 2^kLazy: below that the
      // probabilities stay <= 2^kLazy (exact range for fp16 P and the fp32
      // sums), and the output needs no rescale.
      const float m_cand = fmaxf(m, mx * a.scale_log2);
      const float m_new = (m == -INFINITY || m_cand > m + kSpLazy) ? m_cand : m;
      const float alpha = (m == -INFINITY) ? (m_new == -INFINITY ? 1.f : 0.f) : exp2f(m - m_new);
      uint32_t packed[32];
      float ps[4] = {0.f, 0.f, 0.f, 0.f};  // four independent partial sums
      if (full) {
#pragma unroll
        for (int k = 0; k < 64; k += 2) {
          const float p0 = ex2_approx(sc[k] * a.scale_log2 - m_new);
          const float p1 = ex2_approx(sc[k + 1] * a.scale_log2 - m_new);
          ps[(k >> 1) & 3] += p0 + p1;
          const __half2 ph = __floats2half2_rn(p0, p1);
          packed[k / 2] = *reinterpret_cast<const uint32_t*>(&ph);
        }
      } else {
        const int kme = key0 + hf * 64;
#pragma unroll
        for (int k = 0; k < 64; k += 2) {
          const float p0 = (kme + k < lim && m_new != -INFINITY) ? ex2_approx(sc[k] * a.scale_log2 - m_new) : 0.f;
          const float p1 =
              (kme + k + 1 < lim && m_new != -INFINITY) ? ex2_approx(sc[k + 1] * a.scale_log2 - m_new) : 0.f;
          ps[(k >> 1) & 3] += p0 + p1;
          const __half2 ph = __floats2half2_rn(p0, p1);
          packed[k / 2] = *reinterpret_cast<const uint32_t*>(&ph);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_empty[st]);
      if (c > 0) {
        if (!mbar_wait(pv_done, (c - 1) & 1, a.status, sabort)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (__any_sync(0xffffffffu, alpha != 1.0f)) {
          float o[64];
          tmem_ld64(tmem + lane_off + 256u + static_cast<uint32_t>(hf * 64), o);
#pragma unroll
          for (int k = 0; k < 64; ++k) o[k] *= alpha;
#pragma unroll
          for (int k = 0; k < 64; k += 16) tmem_st16_nowait(tmem + lane_off + 256u + hf * 64 + k, o + k);
          tmem_wait_st();
        }
      }
      // P of this warp's 64 keys into TMEM columns kSpColP + 32 hf .. + 31
      tmem_st16u_nowait(tmem + lane_off + kSpColP + hf * 32, packed);
      tmem_st16u_nowait(tmem + lane_off + kSpColP + hf * 32 + 16, packed + 16);
      tmem_wait_st();  // P (and any rescaled O) in TMEM
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
      l = l * alpha + ((ps[0] + ps[1]) + (ps[2] + ps[3]));
      m = m_new;
    }
    const bool have = ok && nc > 0 && mbar_wait(pv_done, (nc - 1) & 1, a.status, sabort);
    sLh[hf * 128 + row] = l;
    named_bar_sync(1, kSpSoftmax);
    l = sLh[row] + sLh[128 + row];
    if constexpr (kCL > 0) {
      // ------------------------------------------------------ cluster merge
      // This CTA's O / l of row `row` (features 64 hf .. 64 hf + 63) as fp16
      // (|O / l| <= max |v|) and (m, l) into shared memory (the key stages
      // are free), 16-byte pieces of a 256-byte row at piece ^ (row & 15)
      // (conflict-free for lanes = rows); then one bulk copy per owner CTA
      // of its RPC rows into that CTA's slot for this source, counted on its
      // receive barrier.  CTAs without keys send nothing and every owner
      // expects the min(kCL, chunks) CTAs that have keys.  Each CTA then
      // combines its RPC rows over the sources in source order.
      constexpr int RPC = 128 / kCL;
      constexpr uint32_t kSendO = RPC * 256, kSendML = RPC * 8;
      const int crank = sp;
      const int n_src = min(kCL, n_all);
      uint8_t* sSend = sK;                                           // [128][256 B]
      float2* sSendML = reinterpret_cast<float2*>(sK + 128 * 256);  // [128]
      if (nc > 0) {
        float o[64];
        if (have) {
          tc_fence_after();
          tmem_ld64(tmem + lane_off + kSpColO + static_cast<uint32_t>(hf * 64), o);
        } else {
#pragma unroll
          for (int k = 0; k < 64; ++k) o[k] = 0.f;
        }
        const float inv_l = (have && l > 0.f) ? 1.0f / l : 0.f;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const __half2 h = __floats2half2_rn(o[8 * q + 2 * e] * inv_l, o[8 * q + 2 * e + 1] * inv_l);
            w[e] = *reinterpret_cast<const uint32_t*>(&h);
          }
          *reinterpret_cast<uint4*>(sSend + row * 256 + (((hf * 8 + q) ^ (row & 15)) << 4)) =
              make_uint4(w[0], w[1], w[2], w[3]);
        }
        if (hf == 0) sSendML[row] = (have && l > 0.f) ? make_float2(m, l) : make_float2(-INFINITY, 0.f);
        fence_proxy_async_smem();
      }
      named_bar_sync(1, kSpSoftmax);
      __syncwarp();
      cluster_wait();  // every CTA of the cluster runs, its receive barrier initialised
      const int et = threadIdx.x - 64;
      if (nc > 0 && et < kCL) {
        const uint32_t rb = map_to_cta(smem_u32(recv_full), et);
        bulk_s2s_cluster(map_to_cta(smem_u32(smem + oSpRecv) + crank * kSendO, et), sSend + et * kSendO, kSendO, rb);
        bulk_s2s_cluster(map_to_cta(smem_u32(smem + oSpRecvML) + crank * kSendML, et), sSendML + et * RPC, kSendML,
                         rb);
        bulk_commit();
      }
      const bool got = mbar_wait(recv_full, 0, a.status, sabort);
      constexpr int TPR = kSpSoftmax / RPC;  // threads per merged row
      constexpr int FPT = 128 / TPR;         // features per thread
      const int rl = et / TPR, f0 = (et % TPR) * FPT;
      const int r = crank * RPC + rl;        // row of the tile
      const uint8_t* rO = smem + oSpRecv;
      const float2* rML = reinterpret_cast<const float2*>(smem + oSpRecvML);
      // piece of features f0.. in a row sent as tile row r, and the offset in it
      const int piece = ((f0 >> 3) ^ (r & 15)) << 4, poff = (f0 & 7) * 2;
      float M = -INFINITY;
      for (int q = 0; q < n_src; ++q) M = fmaxf(M, rML[q * RPC + rl].x);
      float acc[FPT];
#pragma unroll
      for (int k = 0; k < FPT; ++k) acc[k] = 0.f;
      float wsum = 0.f;
      if (got && M != -INFINITY) {
#pragma unroll 4
        for (int q = 0; q < n_src; ++q) {
          const float2 v = rML[q * RPC + rl];
          const float w = v.y > 0.f ? ex2_approx(v.x - M) * v.y : 0.f;
          wsum += w;
          const __half2* src = reinterpret_cast<const __half2*>(rO + (q * RPC + rl) * 256 + piece + poff);
#pragma unroll
          for (int k = 0; k < FPT; k += 2) {
            const float2 f = __half22float2(src[k / 2]);
            acc[k] += w * f.x;
            acc[k + 1] += w * f.y;
          }
        }
      }
      const int tr = t_base + (r >> 3);
      if (tr < a.n_rows) {
        const float inv = wsum > 0.f ? 1.0f / wsum : 0.f;
        bf16* dst_o =
            a.out + ((static_cast<size_t>(a.q_row0) + bidx * a.n_rows + tr) * a.Hq + g * 8 + (r & 7)) * 128 + f0;
#pragma unroll
        for (int k = 0; k < FPT; k += 4) {
          const __nv_bfloat162 b0 = __floats2bfloat162_rn(acc[k] * inv, acc[k + 1] * inv);
          const __nv_bfloat162 b1 = __floats2bfloat162_rn(acc[k + 2] * inv, acc[k + 3] * inv);
          *reinterpret_cast<uint2*>(dst_o + k) =
              make_uint2(*reinterpret_cast<const uint32_t*>(&b0), *reinterpret_cast<const uint32_t*>(&b1));
        }
      }
      // no CTA leaves before its outgoing copies have read their source (its
      // incoming ones have landed: receive barrier above)
      if (nc > 0 && et < kCL) bulk_wait_read_all();
    } else {
    // this split's partial rows: O / l (fp32, each warp its 64 features) and
    // (m, l), l the two halves' sums added in half order
    const size_t pidx = static_cast<size_t>(grp) * S + sp;
    float* prow = part + (pidx * 128 + row) * 128 + hf * 64;
    if (have) {
      tc_fence_after();
      const float inv_l = l > 0.f ? 1.0f / l : 0.f;
      float o[64];
      tmem_ld64(tmem + lane_off + 256u + static_cast<uint32_t>(hf * 64), o);
#pragma unroll
      for (int k = 0; k < 64; k += 4)
        __stcg(reinterpret_cast<float4*>(prow + k),
               make_float4(o[k] * inv_l, o[k + 1] * inv_l, o[k + 2] * inv_l, o[k + 3] * inv_l));
    }
    if (hf == 0) ml[pidx * 128 + row] = (have && l > 0.f) ? make_float2(m, l) : make_float2(-INFINITY, 0.f);
    __threadfence();
    named_bar_sync(1, kSpSoftmax);
    if (threadIdx.x == 64) *sflag = (atomicAdd(&cnt[grp], 1) == S - 1) ? 1 : 0;
    named_bar_sync(1, kSpSoftmax);
    if (*sflag) {
      // ------------------------------------------------------------ merge
      // (m, l) of every split and row into shared memory (the K stages are
      // free now), each row's weights w_q = 2^(m_q - M) l_q in place of m_q;
      // then the partials (independent, coalesced 512-byte loads) summed in
      // split order
      __threadfence();
      if (threadIdx.x == 64) cnt[grp] = 0;  // every split arrived: zero for the next launch
      const int et = threadIdx.x - 64;
      const size_t p0 = static_cast<size_t>(grp) * S;
      float2* sml = reinterpret_cast<float2*>(sK);  // [S][128]
      float* sinv = reinterpret_cast<float*>(sV);   // [128]
      for (int i = et; i < S * 128; i += kSpSoftmax) sml[i] = __ldcg(&ml[p0 * 128 + i]);
      named_bar_sync(1, kSpSoftmax);
      if (et < 128) {
        float M = -INFINITY;
        for (int q = 0; q < S; ++q) M = fmaxf(M, sml[q * 128 + et].x);
        float wsum = 0.f;
        for (int q = 0; q < S; ++q) {
          const float2 v = sml[q * 128 + et];
          const float w = v.y > 0.f ? ex2_approx(v.x - M) * v.y : 0.f;
          sml[q * 128 + et].x = w;
          wsum += w;
        }
        sinv[et] = wsum > 0.f ? 1.0f / wsum : 0.f;
      }
      named_bar_sync(1, kSpSoftmax);
      // warp w merges rows 16w .. 16w+15, eight rows at a time, so each warp
      // keeps 8 (x 2 splits) independent loads in flight
      constexpr int kRB = 8;
      const int wq = et >> 5;
#pragma unroll 1
      for (int r0 = wq * 16; r0 < wq * 16 + 16; r0 += kRB) {
        float4 acc[kRB];
#pragma unroll
        for (int j = 0; j < kRB; ++j) acc[j] = make_float4(0.f, 0.f, 0.f, 0.f);
        const float4* src = reinterpret_cast<const float4*>(part + (p0 * 128 + r0) * 128) + lane;
#pragma unroll 2
        for (int q = 0; q < S; ++q) {
          float4 f[kRB];
#pragma unroll
          for (int j = 0; j < kRB; ++j) f[j] = __ldcg(src + (static_cast<size_t>(q) * 128 + j) * 32);
#pragma unroll
          for (int j = 0; j < kRB; ++j) {
            const float w = sml[q * 128 + r0 + j].x;
            acc[j].x += w * f[j].x;
            acc[j].y += w * f[j].y;
            acc[j].z += w * f[j].z;
            acc[j].w += w * f[j].w;
          }
        }
#pragma unroll
        for (int j = 0; j < kRB; ++j) {
          const int r = r0 + j;
          const int tr = t_base + (r >> 3);
          if (tr < a.n_rows) {
            const float inv = sinv[r];
            bf16* dst =
                a.out + ((static_cast<size_t>(a.q_row0) + bidx * a.n_rows + tr) * a.Hq + g * 8 + (r & 7)) * 128 +
                lane * 4;
            const __nv_bfloat162 b0 = __floats2bfloat162_rn(acc[j].x * inv, acc[j].y * inv);
            const __nv_bfloat162 b1 = __floats2bfloat162_rn(acc[j].z * inv, acc[j].w * inv);
            *reinterpret_cast<uint2*>(dst) =
                make_uint2(*reinterpret_cast<const uint32_t*>(&b0), *reinterpret_cast<const uint32_t*>(&b1));
          }
        }
      }
    }
    }
  }
  if constexpr (kCL > 0) {
    // the loader, MMA and conversion warps take part in the cluster barrier
    // the softmax warps pass before their sends
    if (warp < 2 || warp >= 10) {
      __syncwarp();
      cluster_wait();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kSpTmem);
  }
}

// S CTAs per (batch entry, row group, KV head); scratch from
// attn_split_scratch_bytes(n_batch * n_groups * Hkv, S), counters zero.
cudaError_t launch_attn_split(const CUtensorMap& mapQ, const CUtensorMap& mapK, const CUtensorMap& mapV,
                              const AttnArgs& a, int S, void* scratch, bool pdl, cudaStream_t s) {
  if (S < 1 || S > 64 || !scratch) return cudaErrorInvalidValue;
  static bool attr_set[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
  if (dev < 0 || dev >= 64 || !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(attn_split_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSpSmem);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) attr_set[dev] = true;
  }
  const int n_groups = (a.n_rows + 15) / 16;
  const int groups_total = a.n_batch * n_groups * a.Hkv;
  const size_t part = static_cast<size_t>(groups_total) * S * 128 * 128 * 4;
  const size_t ml = static_cast<size_t>(groups_total) * S * 128 * 8;
  uint8_t* base = static_cast<uint8_t*>(scratch);
  float* p = reinterpret_cast<float*>(base);
  float2* m = reinterpret_cast<float2*>(base + (part + 255) / 256 * 256);
  int* c = reinterpret_cast<int*>(base + (part + 255) / 256 * 256 + (ml + 255) / 256 * 256);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(S, a.Hkv, a.n_batch * n_groups);
  cfg.blockDim = dim3(kSpThreads);
  cfg.dynamicSmemBytes = kSpSmem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, attn_split_kernel<0>, mapQ, mapK, mapV, mapK, mapV, a, p, m, c);
}

template <int CL>
static cudaError_t split_cl_attr() {
  cudaError_t e = cudaFuncSetAttribute(attn_split_kernel<CL>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSpSmem);
  if (e == cudaSuccess && CL > 8)
    e = cudaFuncSetAttribute(attn_split_kernel<CL>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  return e;
}

// One cluster of cs CTAs (8 or 16) per (batch entry, row group, KV head);
// no scratch.
static cudaError_t split_cl_launch(const CUtensorMap& mapQ, const CUtensorMap& mapK, const CUtensorMap& mapV,
                                   const CUtensorMap& mapKs, const CUtensorMap& mapVs, const AttnArgs& a, int cs,
                                   bool pdl, cudaStream_t s) {
  if (cs != 8 && cs != 16) return cudaErrorInvalidValue;
  static bool attr_set[2][64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
  const int ci = cs == 16 ? 1 : 0;
  if (dev < 0 || dev >= 64 || !attr_set[ci][dev]) {
    cudaError_t e = cs == 16 ? split_cl_attr<16>() : split_cl_attr<8>();
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) attr_set[ci][dev] = true;
  }
  const int n_groups = (a.n_rows + 15) / 16;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(cs, a.Hkv, a.n_batch * n_groups);
  cfg.blockDim = dim3(kSpThreads);
  cfg.dynamicSmemBytes = kSpSmem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = cs;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  if (cs == 16)
    return cudaLaunchKernelEx(&cfg, attn_split_kernel<16>, mapQ, mapK, mapV, mapKs, mapVs, a,
                              static_cast<float*>(nullptr), static_cast<float2*>(nullptr), static_cast<int*>(nullptr));
  return cudaLaunchKernelEx(&cfg, attn_split_kernel<8>, mapQ, mapK, mapV, mapKs, mapVs, a,
                            static_cast<float*>(nullptr), static_cast<float2*>(nullptr), static_cast<int*>(nullptr));
}

cudaError_t launch_attn_split_cl(const CUtensorMap& mapQ, const CUtensorMap& mapK, const CUtensorMap& mapV,
                                 const AttnArgs& a, int cs, bool pdl, cudaStream_t s) {
  if (a.cand_B > 0) return cudaErrorInvalidValue;
  return split_cl_launch(mapQ, mapK, mapV, mapK, mapV, a, cs, pdl, s);
}

cudaError_t launch_attn_cand_cl(const CUtensorMap& mapQ, const CUtensorMap& mapK, const CUtensorMap& mapV,
                                const CUtensorMap& mapKs, const CUtensorMap& mapVs, const AttnArgs& a, int cs,
                                cudaStream_t s) {
  if (a.cand_B < 1 || a.cand_B > 16 || a.n_rows != a.cand_B || a.n_clean != 0 || a.n_batch != a.cand_B ||
      !a.d_len || a.block_table || a.len_sub || a.side_n < 64 * a.cand_B)
    return cudaErrorInvalidValue;
  return split_cl_launch(mapQ, mapK, mapV, mapKs, mapVs, a, cs, false, s);
}

// Clusters of cs CTAs of the cluster-merge form that can be resident at once
// (0: cannot launch).
int attn_split_cl_max_clusters(int cs) {
  if ((cs == 16 ? split_cl_attr<16>() : split_cl_attr<8>()) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(cs, 2, 1);
  cfg.blockDim = dim3(kSpThreads);
  cfg.dynamicSmemBytes = kSpSmem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cs;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  const cudaError_t e = cs == 16 ? cudaOccupancyMaxActiveClusters(&n, attn_split_kernel<16>, &cfg)
                                 : cudaOccupancyMaxActiveClusters(&n, attn_split_kernel<8>, &cfg);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return n;
}

}  // namespace dvlm
