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
// to bf16 for the second product.  The keys are split over an 8-CTA cluster;
// the partial (max, sum, O) of the 8 CTAs are merged through distributed
// shared memory, so there is no second kernel and no global scratch.
#include "kernels.h"
#include "mainloop.cuh"

namespace dvlm {

namespace {
constexpr int kCS = 8;           // CTAs per cluster (key splits)
constexpr int kChunk = 64;       // keys per chunk
constexpr int kTmemCols = 256;   // S: 2 x 64 columns, O: 128 columns
constexpr int kQBytes = 32768;   // 128 rows x 128 d
constexpr int kKBytes = 16384;   // 64 keys x 128 d
constexpr int kVBytes = 16384;   // 128 d x 64 keys
constexpr int kPBytes = 16384;   // 128 rows x 64 keys
constexpr int oQ = 0;
constexpr int oK = oQ + kQBytes;
constexpr int oV = oK + 2 * kKBytes;
constexpr int oP = oV + 2 * kVBytes;
constexpr int oML = oP + 2 * kPBytes;      // m[128], l[128]
constexpr int oBar = oML + 2 * 128 * 4;
constexpr int oMisc = oBar + 16 * 8;
constexpr int kSmem = oMisc + 64 + 1024;
constexpr uint32_t kIdescS = idesc_bf16_f32(128, kChunk);
constexpr uint32_t kIdescO = idesc_bf16_f32(128, 128);
}  // namespace

__global__ void __cluster_dims__(kCS, 1, 1) __launch_bounds__(192, 1)
    attn_bf16_kernel(const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapK,
                     const __grid_constant__ CUtensorMap mapV, const AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sQ = smem + oQ;
  uint8_t* sK = smem + oK;
  uint8_t* sV = smem + oV;
  uint8_t* sP = smem + oP;
  float* sO = reinterpret_cast<float*>(smem + oK);  // reused after the key loop: [128][128]
  float* sM = reinterpret_cast<float*>(smem + oML);
  float* sL = sM + 128;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + oBar);
  uint64_t* q_full = bars;
  uint64_t* kv_full = bars + 1;    // [2]
  uint64_t* kv_empty = bars + 3;   // [2]
  uint64_t* s_full = bars + 5;     // [2]
  uint64_t* p_full = bars + 7;     // [2]
  uint64_t* pv_done = bars + 9;    // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + oMisc);
  volatile int* sabort = reinterpret_cast<volatile int*>(smem + oMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int crank = static_cast<int>(cluster_ctarank());
  const int g = blockIdx.y;                     // KV head
  const int n_groups = (a.n_rows + 15) / 16;
  const int bidx = blockIdx.z / n_groups;       // batch entry
  const int t_base = (blockIdx.z % n_groups) * 16;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 11; ++i) mbar_init(&bars[i], (i == 7 || i == 8) ? 128 : 1);
    *sabort = 0;
    fence_mbar_init();
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
  griddep_launch_dependents();
  griddep_wait();

  const int L = a.d_len ? *a.d_len : a.L_static;
  const int Ltot = L + a.n_rows;
  // Chunk j of 64 keys belongs to CTA j % 8 (round robin): a row's partial
  // sums then do not depend on how many rows the step has, so a causal row
  // gives bitwise the same output in a 1-row AR pass and a 16-row verify pass.
  const int n_chunks = (Ltot + kChunk - 1) / kChunk;
  const int nc = crank < n_chunks ? (n_chunks - crank + kCS - 1) / kCS : 0;
  const int kv_row0 = (a.kv_base + bidx) * a.Hkv + g;

  if (warp == 0) {
    if (lane == 0 && nc > 0) {
      const uint64_t pol = l2_policy_evict_last();
      mbar_arrive_expect_tx(q_full, kQBytes);
      for (int h = 0; h < 2; ++h)
        tma_load_3d(sQ + h * (kQBytes / 2), &mapQ, q_full, h * 64, g * 8, bidx * a.n_rows + t_base, pol);
      for (int jj = 0; jj < nc; ++jj) {
        const int st = jj & 1;
        if (jj >= 2 && !mbar_wait(&kv_empty[st], ((jj >> 1) - 1) & 1, a.status, sabort)) break;
        mbar_arrive_expect_tx(&kv_full[st], kKBytes + kVBytes);
        const int key0 = (crank + kCS * jj) * kChunk;
        for (int h = 0; h < 2; ++h)
          tma_load_2d(sK + st * kKBytes + h * (kKBytes / 2), &mapK, &kv_full[st], h * 64, kv_row0 * a.Lmax + key0,
                      pol);
        tma_load_2d(sV + st * kVBytes, &mapV, &kv_full[st], key0, kv_row0 * 128, pol);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && nc > 0) {
      auto issue_pv = [&](int j) -> bool {
        const int st = j & 1;
        if (!mbar_wait(&p_full[st], (j >> 1) & 1, a.status, sabort)) return false;
        tc_fence_after();
        const uint32_t pa = smem_u32(sP + st * kPBytes), vb = smem_u32(sV + st * kVBytes);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          umma_bf16_ss(tmem + 128, sdesc_kmajor_sw128(pa + 32 * kk), sdesc_kmajor_sw128(vb + 32 * kk), kIdescO,
                       (j > 0 || kk > 0) ? 1u : 0u);
        umma_commit(&pv_done[st]);
        umma_commit(&kv_empty[st]);
        return true;
      };
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
        if (jj >= 1) ok = issue_pv(jj - 1);
      }
      if (ok) issue_pv(nc - 1);
    }
  } else {
    // ---------------------------------------------------------------- softmax
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const int t = t_base + (row >> 3);
    const int limit = (t < a.n_clean) ? (L + t + 1) : Ltot;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int jj = 0; jj < nc; ++jj) {
      const int st = jj & 1;
      const int key0 = (crank + kCS * jj) * kChunk;
      mbar_wait(&s_full[st], (jj >> 1) & 1, a.status, sabort);
      named_bar_sync(1, 128);
      if (*sabort) {
        ok = false;
        break;
      }
      tc_fence_after();
      float s[kChunk];
#pragma unroll
      for (int c = 0; c < kChunk; c += 16) {
        float tmp[16];
        tmem_ld16(tmem + lane_off + static_cast<uint32_t>(st * kChunk + c), tmp);
#pragma unroll
        for (int k = 0; k < 16; ++k) s[c + k] = tmp[k];
      }
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < kChunk; ++c) {
        s[c] = (key0 + c < limit) ? s[c] * a.scale_log2 : -INFINITY;
        mx = fmaxf(mx, s[c]);
      }
      const float m_new = fmaxf(m, mx);
      float alpha = 1.0f, psum = 0.f;
      uint32_t packed[kChunk / 2];
      if (m_new == -INFINITY) {
#pragma unroll
        for (int c = 0; c < kChunk / 2; ++c) packed[c] = 0u;
      } else {
        alpha = exp2f(m - m_new);
#pragma unroll
        for (int c = 0; c < kChunk; c += 2) {
          const __nv_bfloat162 pb = __floats2bfloat162_rn(exp2f(s[c] - m_new), exp2f(s[c + 1] - m_new));
          const float2 pf = __bfloat1622float2(pb);
          psum += pf.x + pf.y;
          packed[c / 2] = *reinterpret_cast<const uint32_t*>(&pb);
        }
      }
      l = l * alpha + psum;
      // P buffer st is free once PV of chunk jj-2 has completed.
      if (jj >= 2) mbar_wait(&pv_done[st], ((jj >> 1) - 1) & 1, a.status, sabort);
      uint8_t* prow = sP + st * kPBytes + row * 128;
#pragma unroll
      for (int cc = 0; cc < 8; ++cc) {
        const uint4 w = make_uint4(packed[cc * 4 + 0], packed[cc * 4 + 1], packed[cc * 4 + 2], packed[cc * 4 + 3]);
        *reinterpret_cast<uint4*>(prow + ((cc ^ (row & 7)) << 4)) = w;
      }
      // Keys past the end of the valid slots may hold anything (NaN poison
      // included); P is exactly 0 there, but 0 * NaN is NaN, so the value
      // rows of those keys are zeroed before the PV product reads them.
      if (key0 + kChunk > Ltot) {
        mbar_wait(&kv_full[st], (jj >> 1) & 1, a.status, sabort);
        uint8_t* vrow = sV + st * kVBytes + row * 128;  // value feature `row`, 64 keys
        const int valid = Ltot - key0;
        for (int cc = 0; cc < 8; ++cc) {
          if (8 * cc + 7 < valid) continue;
          uint16_t* chunk = reinterpret_cast<uint16_t*>(vrow + ((cc ^ (row & 7)) << 4));
          for (int e = 0; e < 8; ++e)
            if (8 * cc + e >= valid) chunk[e] = 0;
        }
      }
      // tcgen05.ld/st are warp-collective: the rescale runs for the whole warp
      // when any of its rows needs it (alpha == 1 leaves a row unchanged).
      if (jj >= 1 && __any_sync(0xffffffffu, alpha != 1.0f)) {
        mbar_wait(&pv_done[(jj - 1) & 1], ((jj - 1) >> 1) & 1, a.status, sabort);
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < 128; c += 16) {
          float o[16];
          tmem_ld16(tmem + lane_off + 128u + c, o);
#pragma unroll
          for (int k = 0; k < 16; ++k) o[k] *= alpha;
          tmem_st16(tmem + lane_off + 128u + c, o);
        }
      }
      m = m_new;
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&p_full[st]);
    }
    // Final PV done -> unnormalised partial O of this CTA into shared memory
    // (the K/V stages are free by then).
    if (ok && nc > 0) {
      mbar_wait(&pv_done[(nc - 1) & 1], ((nc - 1) >> 1) & 1, a.status, sabort);
    }
    named_bar_sync(1, 128);
    const bool have = ok && nc > 0 && !*sabort;
    if (have) tc_fence_after();
#pragma unroll
    for (int c = 0; c < 128; c += 16) {
      float o[16];
      if (have) {
        tmem_ld16(tmem + lane_off + 128u + c, o);
      } else {
#pragma unroll
        for (int k = 0; k < 16; ++k) o[k] = 0.f;
      }
#pragma unroll
      for (int k = 0; k < 16; ++k) sO[row * 128 + ((c + k + 4 * row) & 127)] = o[k];
    }
    sM[row] = have ? m : -INFINITY;
    sL[row] = have ? l : 0.f;
  }
  tc_fence_before();
  cluster_sync();
  // ---------------------------------------------------------------- merge
  // CTA `crank` combines rows [crank*16, crank*16+16) over the 8 partials.
  if (threadIdx.x >= 64) {
    const int et = threadIdx.x - 64;
    const int r = crank * (128 / kCS) + et / 8;
    const int d0 = (et % 8) * 16;
    const int t = t_base + (r >> 3), hl = r & 7;
    float ms[kCS], M = -INFINITY;
    for (int s2 = 0; s2 < kCS; ++s2) {
      ms[s2] = ld_dsmem_f32(map_to_cta(smem_u32(&sM[r]), s2));
      M = fmaxf(M, ms[s2]);
    }
    float acc[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) acc[k] = 0.f;
    float lsum = 0.f;
    if (M != -INFINITY) {
      for (int s2 = 0; s2 < kCS; ++s2) {
        if (ms[s2] == -INFINITY) continue;
        const float w = exp2f(ms[s2] - M);
        lsum += w * ld_dsmem_f32(map_to_cta(smem_u32(&sL[r]), s2));
#pragma unroll
        for (int k = 0; k < 16; k += 4) {
          // rows are stored rotated by 4*row floats (bank spread); undo it
          const int col = (d0 + k + 4 * r) & 127;
          const float4 f = ld_dsmem_f32x4(map_to_cta(smem_u32(&sO[r * 128 + col]), s2));
          acc[k] += w * f.x;
          acc[k + 1] += w * f.y;
          acc[k + 2] += w * f.z;
          acc[k + 3] += w * f.w;
        }
      }
    }
    if (t < a.n_rows) {
      const float inv = lsum > 0.f ? 1.0f / lsum : 0.f;
      bf16* dst = a.out + ((static_cast<size_t>(bidx) * a.n_rows + t) * a.Hq + g * 8 + hl) * 128 + d0;
      uint32_t w[8];
#pragma unroll
      for (int k = 0; k < 16; k += 2) {
        const __nv_bfloat162 pb = __floats2bfloat162_rn(acc[k] * inv, acc[k + 1] * inv);
        w[k / 2] = *reinterpret_cast<const uint32_t*>(&pb);
      }
      reinterpret_cast<uint4*>(dst)[0] = make_uint4(w[0], w[1], w[2], w[3]);
      reinterpret_cast<uint4*>(dst)[1] = make_uint4(w[4], w[5], w[6], w[7]);
    }
  }
  cluster_sync();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

cudaError_t launch_attn_bf16(const CUtensorMap& mapQ, const CUtensorMap& mapK, const CUtensorMap& mapV,
                             const AttnArgs& a, bool pdl, cudaStream_t s) {
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(attn_bf16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  const int n_groups = (a.n_rows + 15) / 16;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(kCS, a.Hkv, a.n_batch * n_groups);
  cfg.blockDim = dim3(192);
  cfg.dynamicSmemBytes = kSmem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, attn_bf16_kernel, mapQ, mapK, mapV, a);
}

}  // namespace dvlm
