// Block-masked GQA attention against the exact KV cache, bf16, tcgen05.
//
// Visibility [Fast-dVLM technical overview (ocdem.com), section 2.2.1;
// Fast-dVLM walkthrough (itsolotime.com), section 4.1]: a clean row t (slot
// L+t) sees slots 0..L+t (C2C, causal); a noisy row sees every slot
// 0..L+n_rows-1 -- the whole cache of vision, prompt and committed tokens
// (N2C) and its own block in both directions (N2N).
//
// Tiling: one KV head's group of 8 query heads x 16 step rows is a single
// 128-row UMMA tile (rows ordered token-major, head-minor, exactly as a 3-D
// TMA box lands).  S = Q K^T (N = 64 keys) and O += P V (V stored
// value-feature-major so both products read K-major operands) accumulate in
// TMEM; softmax runs in fp32 registers, one thread per row, with P rounded
// to fp16 for the second product (the value tile converted to fp16 too).
// The keys are split over a cluster of 8 or 16 CTAs in 64-key chunks (chunk j
// on CTA j mod cluster size); each CTA pushes its partial rows (max, sum and
// the fp16 output rows divided by their sum) with bulk shared-memory copies to
// the CTA that owns those rows, which merges them in source order, so there is
// no second kernel and no global scratch.  Clusters of 16 CTAs (where the
// device can co-schedule them) put one or two chunks on each CTA at decode
// lengths.
#include <cuda_fp16.h>

#include "kernels.h"
#include "mainloop.cuh"

namespace dvlm {

namespace {
constexpr int kChunk = 64;       // keys per chunk
constexpr int kTmemCols = 256;   // S: 2 x 64 columns, O: 128 columns
constexpr int kQBytes = 32768;   // 128 rows x 128 d
constexpr int kKBytes = 16384;   // 64 keys x 128 d
constexpr int kVBytes = 16384;   // 128 d x 64 keys
constexpr int kPBytes = 16384;   // 128 rows x 64 keys
constexpr int oQ = 0;
constexpr int oK = oQ + kQBytes;
constexpr int oV = oK + 2 * kKBytes;
constexpr int oP = oV + 2 * kVBytes;       // two P buffers: the chunks of a pair
constexpr int kRecvBytes = 128 * 128 * 2;  // partial O rows (fp16) received from the cluster
constexpr int oRecv = oP + 2 * kPBytes;
constexpr int oRecvML = oRecv + kRecvBytes;  // (m, l) received: [sources][rows]
constexpr int oML = oRecvML + 128 * 8;       // (m, l) of this CTA's 128 rows
constexpr int oBar = oML + 128 * 8;
constexpr int oMisc = oBar + 16 * 8;
constexpr int kSmem = oMisc + 64 + 1024;
constexpr uint32_t kIdescS = idesc_bf16_f32(128, kChunk);
// P V runs in fp16: probabilities in [0, 1] keep 11 significant bits instead
// of bf16's 8, and the value tile is converted to fp16 in shared memory
// (exact for |v| within fp16's normal range).
constexpr uint32_t kIdescO = idesc_f16_f32(128, 128);
}  // namespace

template <int kCS>  // CTAs per cluster (key splits)
__global__ void __launch_bounds__(192, 1)
    attn_bf16_kernel(const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapK,
                     const __grid_constant__ CUtensorMap mapV, const AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sQ = smem + oQ;
  uint8_t* sK = smem + oK;
  uint8_t* sV = smem + oV;
  uint8_t* sP = smem + oP;
  __half* sO = reinterpret_cast<__half*>(smem + oK);  // reused after the key loop: [128][128] fp16
  __half* sRecvO = reinterpret_cast<__half*>(smem + oRecv);    // [kCS][128 / kCS rows][128]
  float2* sRecvML = reinterpret_cast<float2*>(smem + oRecvML);  // [kCS][128 / kCS rows]
  float2* sML = reinterpret_cast<float2*>(smem + oML);          // [128]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + oBar);
  uint64_t* q_full = bars;
  uint64_t* kv_full = bars + 1;    // [2] K and V of a chunk landed (stage = chunk & 1)
  uint64_t* kv_empty = bars + 3;   // [2] PV of the chunk in that stage done
  uint64_t* s_full = bars + 5;     // [2] S of the chunk in that TMEM buffer ready
  uint64_t* p_full = bars + 7;     // P of a pair of chunks written (one phase per pair)
  uint64_t* pv_done = bars + 8;    // PV of a pair of chunks done (one phase per pair)
  uint64_t* recv_full = bars + 9;  // every cluster CTA's rows of this CTA landed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + oMisc);
  volatile int* sabort = reinterpret_cast<volatile int*>(smem + oMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int crank = static_cast<int>(cluster_ctarank());
  const int g = blockIdx.y;                     // KV head
  const int n_groups = (a.n_rows + 15) / 16;
  const int bidx = blockIdx.z / n_groups;       // batch entry
  const int t_base = (blockIdx.z % n_groups) * 16;

  constexpr int RPC = 128 / kCS;                  // output rows merged by each CTA
  constexpr uint32_t kSendO = RPC * 128 * 2;      // bytes of partial O per destination
  constexpr uint32_t kSendML = RPC * 8;           // bytes of (m, l) per destination
  if (threadIdx.x == 0) {
    for (int i = 0; i < 10; ++i) mbar_init(&bars[i], i == 7 ? 128 : 1);
    *sabort = 0;
    fence_mbar_init();
    mbar_arrive_expect_tx(recv_full, kCS * (kSendO + kSendML));
    tma_prefetch_map(&mapQ);
    tma_prefetch_map(&mapK);
    tma_prefetch_map(&mapV);
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // Receive barriers initialised cluster-wide before any CTA sends (waited on
  // just before the sends).
  cluster_arrive();

  // The cache length is final before this kernel's predecessor runs (only the
  // end of a forward pass moves it), and so are the cache slots below it: both
  // may be read before waiting for the predecessor.  Slots L.. are written by
  // the QKV projection this kernel follows.
  int L = (a.d_lens ? a.d_lens[bidx] : a.d_len ? *a.d_len : a.L_static) - a.len_sub;
  if (a.block_table && L + a.n_rows > a.max_pages * kChunk) {  // the table cannot hold this length
    record_error(a.status, DVLM_ERR_BOUNDS);
    L = a.max_pages * kChunk - a.n_rows;
  }
  const int Ltot = L + a.n_rows;
  // Chunk j of 64 keys belongs to CTA j % kCS (round robin): a row's partial
  // sums then do not depend on how many rows the step has, so a causal row
  // gives bitwise the same output in a 1-row AR pass and a 16-row verify pass.
  const int n_chunks = (Ltot + kChunk - 1) / kChunk;
  const int nc = crank < n_chunks ? (n_chunks - crank + kCS - 1) / kCS : 0;
  const int kv_row0 = (a.kv_base + bidx) * a.Hkv + g;

  if (warp == 0) {
    if (lane == 0 && nc > 0) {
      const uint64_t pol = l2_policy_evict_last();
      auto load_kv = [&](int jj) {
        const int st = jj & 1;
        const int key0 = (crank + kCS * jj) * kChunk;
        mbar_arrive_expect_tx(&kv_full[st], kKBytes + kVBytes);
        int krow = kv_row0 * a.Lmax + key0, vrow = kv_row0 * 128, vx = key0;
        if (a.block_table) {  // chunk = one 64-slot page
          int page = a.block_table[bidx * a.max_pages + key0 / kChunk];
          if (page < 0 || page >= a.n_pages) {
            record_error(a.status, DVLM_ERR_BOUNDS);
            page = 0;
          }
          const int pe = (a.kv_base * a.n_pages + page) * a.Hkv + g;  // (layer, page, KV head)
          krow = pe * kChunk;
          vrow = pe * 128;
          vx = 0;
        }
        for (int h = 0; h < 2; ++h)
          tma_load_2d(sK + st * kKBytes + h * (kKBytes / 2), &mapK, &kv_full[st], h * 64, krow, pol);
        tma_load_2d(sV + st * kVBytes, &mapV, &kv_full[st], vx, vrow, pol);
      };
      const int first = nc < 2 ? nc : 2;
      bool early[2] = {false, false};
      for (int jj = 0; jj < first; ++jj) {
        if ((crank + kCS * jj + 1) * kChunk <= L) {  // entirely below the cache length
          load_kv(jj);
          early[jj] = true;
        }
      }
      griddep_wait();
      mbar_arrive_expect_tx(q_full, kQBytes);
      for (int h = 0; h < 2; ++h)
        tma_load_3d(sQ + h * (kQBytes / 2), &mapQ, q_full, h * 64, g * 8, bidx * a.n_rows + t_base, pol);
      for (int jj = 0; jj < first; ++jj)
        if (!early[jj]) load_kv(jj);
      for (int jj = 2; jj < nc; ++jj) {
        if (!mbar_wait(&kv_empty[jj & 1], ((jj >> 1) - 1) & 1, a.status, sabort)) break;
        load_kv(jj);
      }
    } else if (lane == 0) {
      griddep_wait();
    }
  } else if (warp == 1) {
    griddep_wait();
    if (lane == 0 && nc > 0) {
      bool ok = mbar_wait(q_full, 0, a.status, sabort);
      for (int jj = 0; ok && jj < nc; ++jj) {
        const int st = jj & 1;
        if (!mbar_wait(&kv_full[st], (jj >> 1) & 1, a.status, sabort)) break;
        tc_fence_after();
        const uint32_t qa = smem_u32(sQ), kb = smem_u32(sK + st * kKBytes);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const int h = kk >> 2, off = (kk & 3) * 32;
          umma_bf16_ss(tmem + st * kChunk, sdesc_kmajor_sw128(qa + h * (kQBytes / 2) + off),
                       sdesc_kmajor_sw128(kb + h * (kKBytes / 2) + off), kIdescS, kk > 0 ? 1u : 0u);
        }
        umma_commit(&s_full[st]);
        if ((jj & 1) == 1 || jj == nc - 1) {  // end of a pair of chunks: their PV products
          if (!mbar_wait(p_full, (jj >> 1) & 1, a.status, sabort)) {
            ok = false;
            break;
          }
          tc_fence_after();
          for (int c = jj & ~1; c <= jj; ++c) {
            const uint32_t pa = smem_u32(sP + (c & 1) * kPBytes), vb = smem_u32(sV + (c & 1) * kVBytes);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_bf16_ss(tmem + 128, sdesc_kmajor_sw128(pa + 32 * kk), sdesc_kmajor_sw128(vb + 32 * kk), kIdescO,
                           (c > 0 || kk > 0) ? 1u : 0u);
            umma_commit(&kv_empty[c & 1]);
          }
          umma_commit(pv_done);
        }
      }
    }
  } else {
    // ---------------------------------------------------------------- softmax
    griddep_wait();
    // The next kernel (the output projection) may launch now and stream its
    // weights on the SMs this kernel leaves idle; it reads this kernel's
    // output only after its own wait (at most two kernels overlap).
    if (threadIdx.x == 64) griddep_launch_dependents();
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const int t = t_base + (row >> 3);
    const int limit = (t < a.n_clean) ? (L + t + 1) : Ltot;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    // Writes P of chunk jj (probabilities exp2(s - m_new), fp16) for this row
    // into the chunk's P buffer and converts this thread's value row of the
    // chunk; returns the row sum of the probabilities.
    auto emit_p = [&](int jj, const float (&sc)[64], float m_new) -> float {
      const int key0 = (crank + kCS * jj) * kChunk;
      uint32_t packed[kChunk / 2];
      float ps[4] = {0.f, 0.f, 0.f, 0.f};
      if (m_new == -INFINITY) {
#pragma unroll
        for (int c = 0; c < kChunk / 2; ++c) packed[c] = 0u;
      } else {
#pragma unroll
        for (int c = 0; c < kChunk; c += 2) {
          const float p0 = ex2_approx(sc[c] - m_new), p1 = ex2_approx(sc[c + 1] - m_new);
          ps[(c >> 1) & 3] += p0 + p1;
          const __half2 ph = __floats2half2_rn(p0, p1);
          packed[c / 2] = *reinterpret_cast<const uint32_t*>(&ph);
        }
      }
      const float psum = (ps[0] + ps[1]) + (ps[2] + ps[3]);
      uint8_t* prow = sP + (jj & 1) * kPBytes + row * 128;
#pragma unroll
      for (int cc = 0; cc < 8; ++cc) {
        const uint4 w = make_uint4(packed[cc * 4 + 0], packed[cc * 4 + 1], packed[cc * 4 + 2], packed[cc * 4 + 3]);
        *reinterpret_cast<uint4*>(prow + ((cc ^ (row & 7)) << 4)) = w;
      }
      // Value row `row` of this chunk (64 keys) to fp16 in place; keys past
      // the valid slots may hold anything (NaN poison included) and 0 * NaN
      // is NaN, so they become 0.
      {
        const int st = jj & 1;
        mbar_wait(&kv_full[st], (jj >> 1) & 1, a.status, sabort);
        uint8_t* vrow = sV + st * kVBytes + row * 128;
        const int valid = Ltot - key0;
#pragma unroll
        for (int cc = 0; cc < 8; ++cc) {
          uint4* p16 = reinterpret_cast<uint4*>(vrow + ((cc ^ (row & 7)) << 4));
          uint4 w = *p16;
          uint32_t* wv = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wv[e]));
            const int k0 = 8 * cc + 2 * e;
            const __half2 h = __floats2half2_rn(k0 < valid ? f.x : 0.f, k0 + 1 < valid ? f.y : 0.f);
            wv[e] = *reinterpret_cast<const uint32_t*>(&h);
          }
          *p16 = w;
        }
      }
      return psum;
    };
    auto load_scores = [&](int jj, float (&sc)[64]) -> float {
      const int key0 = (crank + kCS * jj) * kChunk;
      tmem_ld64(tmem + lane_off + static_cast<uint32_t>((jj & 1) * kChunk), sc);
      float mq[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int c = 0; c < kChunk; ++c) {
        sc[c] = (key0 + c < limit) ? sc[c] * a.scale_log2 : -INFINITY;
        mq[c & 3] = fmaxf(mq[c & 3], sc[c]);
      }
      return fmaxf(fmaxf(mq[0], mq[1]), fmaxf(mq[2], mq[3]));
    };
    for (int jj0 = 0; jj0 < nc; jj0 += 2) {
      const bool two = jj0 + 1 < nc;
      mbar_wait(&s_full[0], (jj0 >> 1) & 1, a.status, sabort);
      if (two) mbar_wait(&s_full[1], (jj0 >> 1) & 1, a.status, sabort);
      named_bar_sync(1, 128);
      if (*sabort) {
        ok = false;
        break;
      }
      tc_fence_after();
      // Pass 1: row maxima of the pair (scores re-read from TMEM in pass 2,
      // so at most one chunk's scores occupy registers at a time).
      float mx;
      {
        float sc[64];
        mx = load_scores(jj0, sc);
        if (two) mx = fmaxf(mx, load_scores(jj0 + 1, sc));
      }
      const float m_new = fmaxf(m, mx);
      const float alpha = (m_new == -INFINITY) ? 1.0f : exp2f(m - m_new);
      if (jj0 > 0) {
        // the previous pair's products are complete: O is stable, P is free
        mbar_wait(pv_done, ((jj0 >> 1) - 1) & 1, a.status, sabort);
        tc_fence_after();
        // tcgen05.ld/st are warp-collective: rescale the whole warp when any
        // of its rows needs it (alpha == 1 leaves a row unchanged)
        if (__any_sync(0xffffffffu, alpha != 1.0f)) {
#pragma unroll 1
          for (int c = 0; c < 128; c += 64) {
            float o[64];
            tmem_ld64(tmem + lane_off + 128u + c, o);
#pragma unroll
            for (int k = 0; k < 64; ++k) o[k] *= alpha;
#pragma unroll
            for (int k = 0; k < 64; k += 16) tmem_st16_nowait(tmem + lane_off + 128u + c + k, o + k);
            tmem_wait_st();
          }
        }
      }
      // Pass 2: probabilities of each chunk into the P buffer.
      float psum;
      {
        float sc[64];
        load_scores(jj0, sc);
        psum = emit_p(jj0, sc, m_new);
      }
      if (two) {
        float sc[64];
        load_scores(jj0 + 1, sc);
        psum += emit_p(jj0 + 1, sc, m_new);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(p_full);
      l = l * alpha + psum;
      m = m_new;
    }
    // Final PV done -> unnormalised partial O of this CTA into shared memory
    // (the K/V stages are free by then).
    if (ok && nc > 0) mbar_wait(pv_done, ((nc - 1) >> 1) & 1, a.status, sabort);
    named_bar_sync(1, 128);
    const bool have = ok && nc > 0 && !*sabort;
    if (have) tc_fence_after();
    // Partial O row `row`, divided by its own sum l (|O / l| <= max |v|), as
    // fp16: 16 chunks of 8 values, chunk c8 stored at slot c8 ^ (row & 15)
    // (conflict-free here, lanes = rows, and in the merge's reads).
    uint4* sO16 = reinterpret_cast<uint4*>(sO);
    const float inv_l = (have && l > 0.f) ? 1.0f / l : 0.f;
#pragma unroll
    for (int c = 0; c < 128; c += 64) {
      float o[64];
      if (have) {
        tmem_ld64(tmem + lane_off + 128u + c, o);
      } else {
#pragma unroll
        for (int k = 0; k < 64; ++k) o[k] = 0.f;
      }
#pragma unroll
      for (int k = 0; k < 64; k += 8) {
        uint32_t w[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const __half2 h = __floats2half2_rn(o[k + 2 * q] * inv_l, o[k + 2 * q + 1] * inv_l);
          w[q] = *reinterpret_cast<const uint32_t*>(&h);
        }
        const int c8 = (c + k) >> 3;
        sO16[row * 16 + (c8 ^ (row & 15))] = make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
    sML[row] = have ? make_float2(m, l) : make_float2(-INFINITY, 0.f);
    // Rows [d*RPC, (d+1)*RPC) of the partial go to cluster CTA d, which merges
    // them: copies by the bulk-copy engine into that CTA's receive buffer,
    // counted on its receive barrier.
    fence_proxy_async_smem();
    named_bar_sync(1, 128);
    cluster_wait();
    if (warp == 2 && lane < kCS) {
      const uint32_t rb = map_to_cta(smem_u32(recv_full), lane);
      bulk_s2s_cluster(map_to_cta(smem_u32(sRecvO) + crank * kSendO, lane), sO + lane * RPC * 128, kSendO, rb);
      bulk_s2s_cluster(map_to_cta(smem_u32(sRecvML) + crank * kSendML, lane), sML + lane * RPC, kSendML, rb);
      bulk_commit();
    }
  }
  if (warp < 2) {
    __syncwarp();
    cluster_wait();
  }
  // Every CTA has issued its copies once all have arrived here: a CTA leaves
  // only after that (second barrier, waited on at exit).
  __syncwarp();
  cluster_arrive();
  // ---------------------------------------------------------------- merge
  // CTA `crank` combines rows [crank*RPC, (crank+1)*RPC) over the kCS partials,
  // read from its own receive buffer in source order.
  if (threadIdx.x >= 64) {
    constexpr int TPR = 128 / RPC;  // threads per row
    constexpr int DPT = 128 / TPR;  // value features per thread
    const int et = threadIdx.x - 64;
    const int rl = et / TPR;
    const int r = crank * RPC + rl;
    const int d0 = (et % TPR) * DPT;
    const int t = t_base + (r >> 3), hl = r & 7;
    const bool got = mbar_wait(recv_full, 0, a.status, sabort);
    float M = -INFINITY;
#pragma unroll
    for (int s2 = 0; s2 < kCS; ++s2) M = fmaxf(M, sRecvML[s2 * RPC + rl].x);
    float acc[DPT];
#pragma unroll
    for (int k = 0; k < DPT; ++k) acc[k] = 0.f;
    float lsum = 0.f;
    if (got && M != -INFINITY) {
      // weight of each partial: its sum l at the common maximum (0 for a
      // source without keys for this row)
      float w[kCS];
#pragma unroll
      for (int s2 = 0; s2 < kCS; ++s2) {
        const float2 ml = sRecvML[s2 * RPC + rl];
        w[s2] = ml.x == -INFINITY ? 0.f : ex2_approx(ml.x - M) * ml.y;
      }
      const uint4* rO16 = reinterpret_cast<const uint4*>(sRecvO);
#pragma unroll
      for (int k = 0; k < DPT / 8; ++k) {
        const int c8 = (d0 >> 3) + k;
        uint4 v[kCS];
#pragma unroll
        for (int s2 = 0; s2 < kCS; ++s2) v[s2] = rO16[(s2 * RPC + rl) * 16 + (c8 ^ (r & 15))];
#pragma unroll
        for (int s2 = 0; s2 < kCS; ++s2) {
          const uint32_t* vw = reinterpret_cast<const uint32_t*>(&v[s2]);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&vw[q]));
            acc[8 * k + 2 * q] += w[s2] * f.x;
            acc[8 * k + 2 * q + 1] += w[s2] * f.y;
          }
        }
      }
#pragma unroll
      for (int s2 = 0; s2 < kCS; ++s2) lsum += w[s2];
    }
    if (t < a.n_rows) {
      const float inv = lsum > 0.f ? 1.0f / lsum : 0.f;
      bf16* dst = a.out + ((static_cast<size_t>(bidx) * a.n_rows + t) * a.Hq + g * 8 + hl) * 128 + d0;
#pragma unroll
      for (int k = 0; k < DPT; k += 8) {
        uint32_t w[4];
#pragma unroll
        for (int q = 0; q < 8; q += 2) {
          const __nv_bfloat162 pb = __floats2bfloat162_rn(acc[k + q] * inv, acc[k + q + 1] * inv);
          w[q / 2] = *reinterpret_cast<const uint32_t*>(&pb);
        }
        reinterpret_cast<uint4*>(dst + k)[0] = make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
  }
  if (warp == 2 && lane < kCS) bulk_wait_read_all();
  // No CTA leaves while a copy into or out of its shared memory may run: its
  // own incoming copies landed (receive barrier), its outgoing ones have read
  // their source, and every other CTA has issued its copies.
  tc_fence_before();
  cluster_wait();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int CS>
static cudaError_t attn_launch(const CUtensorMap& mapQ, const CUtensorMap& mapK, const CUtensorMap& mapV,
                               const AttnArgs& a, bool pdl, cudaStream_t s) {
  // function attributes are per device: set once on each device that launches
  static bool attr_set[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
  if (dev < 0 || dev >= 64 || !attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(attn_bf16_kernel<CS>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    if (e != cudaSuccess) return e;
    if (CS > 8) {
      e = cudaFuncSetAttribute(attn_bf16_kernel<CS>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
      if (e != cudaSuccess) return e;
    }
    if (dev >= 0 && dev < 64) attr_set[dev] = true;
  }
  const int n_groups = (a.n_rows + 15) / 16;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(CS, a.Hkv, a.n_batch * n_groups);
  cfg.blockDim = dim3(192);
  cfg.dynamicSmemBytes = kSmem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = CS;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, attn_bf16_kernel<CS>, mapQ, mapK, mapV, a);
}

cudaError_t launch_attn_bf16(const CUtensorMap& mapQ, const CUtensorMap& mapK, const CUtensorMap& mapV,
                             const AttnArgs& a, bool pdl, cudaStream_t s, int cs) {
  return launch_attn_split_cl(mapQ, mapK, mapV, a, cs, pdl, s);
}

// Clusters of cs CTAs that can be resident at once (0: cannot launch).
int attn_max_clusters(int cs) {
  return attn_split_cl_max_clusters(cs);
  auto kern = cs == 16 ? attn_bf16_kernel<16> : attn_bf16_kernel<8>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem) != cudaSuccess ||
      (cs > 8 && cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess)) {
    cudaGetLastError();
    return 0;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(cs, 2, 1);
  cfg.blockDim = dim3(192);
  cfg.dynamicSmemBytes = kSmem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cs;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return n;
}

}  // namespace dvlm
