// Stage 2 kernel: block-sparse attention forward on sm_100a (tcgen05 + TMA + TMEM),
// with the online-softmax-aware P.V skip.
//
// Stage 2 of the SpargeAttn abstract: the attention is computed only on the kept
// blocks ("skip of some matrix multiplications"), and an online-softmax-aware
// filter skips more P.V products at no extra cost. The DynSparse article places
// the selection inside the FlashAttention operator; this kernel is that operator.
//
// One CTA = one 128-row query tile = query blocks (2t, 2t+1) of one head. The
// tile walks the ascending union of the two blocks' kept key blocks; the half
// that did not keep a block sees -inf scores for it, so each 64-row query block
// gets exactly its own mask. Per key block j (64 keys):
//   S = Q K_j^T          128x64 fp32 in TMEM (tcgen05.mma, both operands TMA'd
//                        into 128B-swizzled shared memory)
//   softmax warps        read S from TMEM (one thread per row), scale/mask, row max,
//                        lambda vote per 64-row half, exp2, row sum, P -> bf16 in
//                        shared memory (128B-swizzled, K-major)
//   O += P V_j           128xD fp32 in TMEM (V read as an MN-major operand)
// Roles: warp 0 = TMA producer, warp 1 = MMA issuer (one thread) and TMEM owner,
// warp 2 = builds the union list, warps 4..7 = softmax / correction / epilogue.
// S is double-buffered in TMEM so S(j+1) overlaps the softmax of S(j).
// The running max used for the exponentials is raised lazily (only when a row's
// max grows by more than 2^8), which leaves O/l unchanged; the lambda test uses
// the exact running max.
#pragma once

#include "sa_device.cuh"

namespace sa {

template <int D, int ST>
struct FwdCfg {
  static constexpr int kRows = 128;                    // query rows per tile
  static constexpr int kChunks = D / 64;               // 128-byte (64 x bf16) column chunks
  static constexpr int kQChunkBytes = kRows * 128;     // 16 KB
  static constexpr int kKVChunkBytes = kBlock * 128;   // 8 KB
  static constexpr int kQBytes = kChunks * kQChunkBytes;
  static constexpr int kKVBytes = kChunks * kKVChunkBytes;
  static constexpr int kPBytes = kRows * 128;          // 128 x 64 bf16
  // shared-memory layout (offsets from a 1024-aligned base)
  static constexpr int oQ = 0;
  static constexpr int oK = oQ + kQBytes;
  static constexpr int oV = oK + ST * kKVBytes;
  static constexpr int oP = oV + ST * kKVBytes;
  static constexpr int oBar = oP + kPBytes;            // mbarriers
  static constexpr int kNumBars = 2 * ST + 9;
  static constexpr int oMisc = oBar + kNumBars * 8;    // small words
  static constexpr int oList = oMisc + 64;
  static constexpr int kSmemBytes = oList + kMaxNb * 4 + 1024;  // + alignment slack
  // TMEM columns
  static constexpr uint32_t kColS0 = 0, kColS1 = 64, kColO = 128;
  static constexpr uint32_t kTmemCols = 256;
  static constexpr uint32_t kIdescS = idesc_bf16_f32(128, 64, false);
  static constexpr uint32_t kIdescPV = idesc_bf16_f32(128, D, true);
};

template <int D, int ST>
__global__ void __launch_bounds__(256, 1)
    fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const uint8_t* __restrict__ mask,
               const int* __restrict__ work, __nv_bfloat16* __restrict__ O, int N, int Nb, int Tq,
               long long num_tiles, float scale_log2, float lam_log2, int lam_on, int causal,
               unsigned long long* __restrict__ stats) {
  using C = FwdCfg<D, ST>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = base + C::oQ;
  uint8_t* sK = base + C::oK;
  uint8_t* sV = base + C::oV;
  uint8_t* sP = base + C::oP;
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + C::oBar);
  uint64_t* full = bars;               // [ST] K/V stage loaded
  uint64_t* empty = bars + ST;         // [ST] K/V stage free
  uint64_t* q_full = bars + 2 * ST;    // Q tile loaded
  uint64_t* s_full = q_full + 1;       // [2] S buffer written by MMA
  uint64_t* s_free = q_full + 3;       // [2] S buffer read by softmax
  uint64_t* p_full = q_full + 5;       // P written (and O corrected)
  uint64_t* pv_done = q_full + 6;      // P.V done (O stable, P buffer free)
  uint64_t* vote_bar = q_full + 7;     // lambda vote of the 4 softmax warps (one phase per entry)
  uint64_t* drain = q_full + 8;        // MMA issuer: all its MMAs finished
  int* misc = reinterpret_cast<int*>(base + C::oMisc);
  volatile int* abort_flag = misc + 0;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(misc + 1);
  int* list_n = misc + 2;
  volatile int* pv_need = misc + 4;    // [2] by k parity: issue P.V for entry k
  volatile int* votes = misc + 8;      // [2][4] by k parity, per softmax warp
  uint32_t* lst = reinterpret_cast<uint32_t*>(base + C::oList);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (blockIdx.x >= num_tiles) return;
  long long tile = work ? static_cast<long long>(work[blockIdx.x]) : static_cast<long long>(blockIdx.x);
  if (tile < 0 || tile >= num_tiles) {  // corrupt work list: record and skip this CTA
    if (threadIdx.x == 0) atomicOr(&g_dev_error, DEVERR_RANGE);
    return;
  }
  const long long bh = tile / Tq;
  const int t = static_cast<int>(tile - bh * Tq);
  const int qb0 = 2 * t, qb1 = 2 * t + 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < ST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(q_full, 1);
    mbar_init(&s_full[0], 1);
    mbar_init(&s_full[1], 1);
    mbar_init(&s_free[0], 128);
    mbar_init(&s_free[1], 128);
    mbar_init(p_full, 128);
    mbar_init(pv_done, 1);
    mbar_init(vote_bar, 4);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  if (warp == 1) tmem_alloc(tmem_holder, C::kTmemCols);
  if (warp == 2) {
    // Ascending union of the kept lists of query blocks qb0 and qb1, with one
    // flag bit per half; causal drops key blocks after the half's query block.
    const uint8_t* m0 = mask + (bh * Nb + qb0) * static_cast<long long>(Nb);
    const uint8_t* m1 = (qb1 < Nb) ? m0 + Nb : nullptr;
    const int jend = causal ? min(Nb, qb1 + 1) : Nb;
    int n = 0;
    for (int jb = 0; jb < jend; jb += 32) {
      const int j = jb + lane;
      uint32_t a = 0, b = 0;
      if (j < jend) {
        a = m0[j] != 0;
        b = (m1 != nullptr) ? (m1[j] != 0) : 0u;
        if (causal) {
          a &= (j <= qb0) ? 1u : 0u;
          b &= (j <= qb1) ? 1u : 0u;
        }
      }
      const uint32_t any = a | b;
      const unsigned bal = __ballot_sync(0xffffffffu, any != 0);
      if (any) lst[n + __popc(bal & ((1u << lane) - 1u))] = static_cast<uint32_t>(j) | (a << 30) | (b << 31);
      n += __popc(bal);
    }
    if (lane == 0) *list_n = n;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const int n = *list_n;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && n > 0) {
      mbar_expect_tx(q_full, C::kQBytes);
#pragma unroll
      for (int c = 0; c < C::kChunks; ++c)
        tma_load_3d(sQ + c * C::kQChunkBytes, &tmQ, c * 64, t * 128, static_cast<int>(bh), q_full);
      int k = 0;
      for (; k < n; ++k) {
        const int s = k % ST;
        const uint32_t round = static_cast<uint32_t>(k / ST);
        if (!mbar_wait(&empty[s], (round & 1u) ^ 1u, abort_flag)) break;
        const int j = static_cast<int>(lst[k] & 0xFFFFu);
        mbar_expect_tx(&full[s], 2 * C::kKVBytes);
#pragma unroll
        for (int c = 0; c < C::kChunks; ++c) {
          tma_load_3d(sK + s * C::kKVBytes + c * C::kKVChunkBytes, &tmK, c * 64, j * kBlock,
                      static_cast<int>(bh), &full[s]);
          tma_load_3d(sV + s * C::kKVBytes + c * C::kKVChunkBytes, &tmV, c * 64, j * kBlock,
                      static_cast<int>(bh), &full[s]);
        }
      }
      // Before leaving, let every load this thread issued land (bounded).
      mbar_wait_drain(q_full, 0u);
      for (int kk = max(0, k - ST); kk < k; ++kk)
        mbar_wait_drain(&full[kk % ST], static_cast<uint32_t>(kk / ST) & 1u);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && n > 0) {
      const uint32_t sQa = smem_u32(sQ), sKa = smem_u32(sK), sVa = smem_u32(sV), sPa = smem_u32(sP);
      bool ok = mbar_wait(q_full, 0u, abort_flag);
      tc_fence_after();
      auto issue_S = [&](int k) -> bool {
        const int s = k % ST, sb = k & 1;
        if (!mbar_wait(&full[s], static_cast<uint32_t>(k / ST) & 1u, abort_flag)) return false;
        if (!mbar_wait(&s_free[sb], (static_cast<uint32_t>(k >> 1) & 1u) ^ 1u, abort_flag)) return false;
        tc_fence_after();
        const uint32_t dS = tmem_base + (sb ? C::kColS1 : C::kColS0);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk & 3) * 32;  // 16 bf16 = 32 bytes inside the swizzle atom
          const uint64_t ad = sdesc_sw128(sQa + (kk >> 2) * C::kQChunkBytes + off, 16, 1024);
          const uint64_t bd = sdesc_sw128(sKa + s * C::kKVBytes + (kk >> 2) * C::kKVChunkBytes + off, 16, 1024);
          tc_mma_ss(dS, ad, bd, C::kIdescS, kk > 0 ? 1u : 0u);
        }
        tc_commit(&s_full[sb]);
        return true;
      };
      if (ok) ok = issue_S(0);
      uint32_t o_init = 0;
      unsigned long long pv_tiles = 0;
      for (int k = 0; ok && k < n; ++k) {
        if (k + 1 < n) {
          if (!issue_S(k + 1)) break;
        }
        if (!mbar_wait(p_full, static_cast<uint32_t>(k) & 1u, abort_flag)) break;
        tc_fence_after();
        const int s = k % ST;
        if (pv_need[k & 1]) {
          const uint32_t dO = tmem_base + C::kColO;
#pragma unroll
          for (int kk = 0; kk < kBlock / 16; ++kk) {
            const uint64_t ad = sdesc_sw128(sPa + kk * 32, 16, 1024);
            const uint64_t bd = sdesc_sw128(sVa + s * C::kKVBytes + kk * 16 * 128, C::kKVChunkBytes, 1024);
            tc_mma_ss(dO, ad, bd, C::kIdescPV, (o_init | static_cast<uint32_t>(kk > 0)));
          }
          o_init = 1u;
          ++pv_tiles;
        }
        tc_commit(pv_done);
        tc_commit(&empty[s]);
      }
      // Drain: wait until every MMA this thread issued has finished (bounded).
      tc_commit(drain);
      mbar_wait_drain(drain, 0u);
      if (stats) {
        atomicAdd(&stats[2], static_cast<unsigned long long>(n));
        atomicAdd(&stats[3], pv_tiles);
      }
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax warps
    const int wq = warp & 3;
    const int row = wq * 32 + lane;          // tile row == TMEM lane
    const int half = row >> 6;
    const long long qrow = static_cast<long long>(t) * 128 + row;
    const bool valid = qrow < N;
    const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(wq * 32) << 16);
    float m_true = -INFINITY, m_ref = -INFINITY, l = 0.f;
    unsigned long long kept_pairs = 0, skipped_pairs = 0;
    bool alive = true;
    uint8_t* prow = sP + row * 128;
    for (int k = 0; k < n; ++k) {
      const uint32_t e = lst[k];
      const int j = static_cast<int>(e & 0xFFFFu);
      const bool keep_lo = (e >> 30) & 1u, keep_hi = (e >> 31) & 1u;
      const bool keep = half ? keep_hi : keep_lo;
      const int sb = k & 1;
      if (!warp_wait(&s_full[sb], static_cast<uint32_t>(k >> 1) & 1u, abort_flag)) { alive = false; break; }
      tc_fence_after();
      float s[64];
      tmem_ld32(lane_base + (sb ? C::kColS1 : C::kColS0), *reinterpret_cast<float(*)[32]>(&s[0]));
      tmem_ld32(lane_base + (sb ? C::kColS1 : C::kColS0) + 32, *reinterpret_cast<float(*)[32]>(&s[32]));
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(&s_free[sb]);

      const bool part = keep && valid;
      const int kbase = j * kBlock;
      // visible columns: c < ncol (tail) and, with causal, kbase + c <= qrow
      int ncol = min(kBlock, N - kbase);
      if (causal) ncol = min(ncol, static_cast<int>(qrow - kbase) + 1);
      if (!part) ncol = 0;
      float rmax = -INFINITY;
#pragma unroll
      for (int c = 0; c < 64; ++c) {
        const float x = (c < ncol) ? s[c] * scale_log2 : -INFINITY;
        s[c] = x;
        rmax = fmaxf(rmax, x);
      }
      // lambda vote: a half skips P.V when all its rows that see the block pass
      bool half_skip = false;
      if (lam_on) {
        const bool pass = !(rmax > -INFINITY) || (rmax - m_true < lam_log2);
        const bool wpass = __all_sync(0xffffffffu, pass);
        if (lane == 0) {
          votes[(k & 1) * 4 + wq] = wpass ? 1 : 0;
          mbar_arrive(vote_bar);
        }
        if (!warp_wait(vote_bar, static_cast<uint32_t>(k) & 1u, abort_flag)) { alive = false; break; }
        half_skip = votes[(k & 1) * 4 + 2 * half] && votes[(k & 1) * 4 + 2 * half + 1];
      }
      const bool contrib_lo = keep_lo && !(lam_on && votes[(k & 1) * 4 + 0] && votes[(k & 1) * 4 + 1]);
      const bool contrib_hi = keep_hi && !(lam_on && votes[(k & 1) * 4 + 2] && votes[(k & 1) * 4 + 3]);

      const float m_new = fmaxf(m_true, rmax);
      float alpha = 1.f;
      const bool raise = m_new > m_ref + 8.f;   // also true for the first finite max
      if (raise) {
        alpha = ex2(m_ref - m_new);             // 0 when m_ref = -inf
        m_ref = m_new;
      }
      m_true = m_new;
      const float mref = (m_ref == -INFINITY) ? 0.f : m_ref;
      float rsum = 0.f;
#pragma unroll
      for (int c = 0; c < 64; ++c) {
        const float p = ex2(s[c] - mref);
        s[c] = p;
        rsum += p;
      }
      l = l * alpha + rsum;
      // P.V of the previous entry must be complete before O and P are touched.
      if (k > 0) {
        if (!warp_wait(pv_done, static_cast<uint32_t>(k - 1) & 1u, abort_flag)) { alive = false; break; }
        tc_fence_after();
        if (__any_sync(0xffffffffu, raise)) {
#pragma unroll
          for (int cc = 0; cc < D; cc += 32) {
            float o[32];
            tmem_ld32(lane_base + C::kColO + cc, o);
            tmem_wait_ld();
#pragma unroll
            for (int x = 0; x < 32; ++x) o[x] *= alpha;
            tmem_st32(lane_base + C::kColO + cc, o);
          }
          tmem_wait_st();
        }
      }
      // P -> bf16, 128B-swizzled K-major rows (16-byte chunk c of row r at c ^ (r & 7)).
      const bool zero_p = half_skip;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        uint4 v;
        if (zero_p) {
          v = make_uint4(0u, 0u, 0u, 0u);
        } else {
          v.x = pack_bf16x2(s[8 * c + 0], s[8 * c + 1]);
          v.y = pack_bf16x2(s[8 * c + 2], s[8 * c + 3]);
          v.z = pack_bf16x2(s[8 * c + 4], s[8 * c + 5]);
          v.w = pack_bf16x2(s[8 * c + 6], s[8 * c + 7]);
        }
        *reinterpret_cast<uint4*>(prow + ((c ^ (row & 7)) << 4)) = v;
      }
      if (threadIdx.x == 128) {
        pv_need[k & 1] = (contrib_lo || contrib_hi) ? 1 : 0;
        kept_pairs += static_cast<unsigned long long>(keep_lo) + static_cast<unsigned long long>(keep_hi);
        skipped_pairs += static_cast<unsigned long long>(keep_lo && !contrib_lo) +
                         static_cast<unsigned long long>(keep_hi && !contrib_hi);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(p_full);
    }
    // ------------------------------------------------------------ epilogue
    if (alive && n > 0) {
      if (warp_wait(pv_done, static_cast<uint32_t>(n - 1) & 1u, abort_flag)) {
        tc_fence_after();
        const float inv = (l > 0.f) ? 1.f / l : 0.f;
        __nv_bfloat16* orow = O + (bh * N + qrow) * static_cast<long long>(D);
#pragma unroll
        for (int cc = 0; cc < D; cc += 32) {
          float o[32];
          tmem_ld32(lane_base + C::kColO + cc, o);
          tmem_wait_ld();
          if (valid) {
#pragma unroll
            for (int x = 0; x < 32; x += 8) {
              uint4 v;
              v.x = pack_bf16x2(l > 0.f ? o[x + 0] * inv : 0.f, l > 0.f ? o[x + 1] * inv : 0.f);
              v.y = pack_bf16x2(l > 0.f ? o[x + 2] * inv : 0.f, l > 0.f ? o[x + 3] * inv : 0.f);
              v.z = pack_bf16x2(l > 0.f ? o[x + 4] * inv : 0.f, l > 0.f ? o[x + 5] * inv : 0.f);
              v.w = pack_bf16x2(l > 0.f ? o[x + 6] * inv : 0.f, l > 0.f ? o[x + 7] * inv : 0.f);
              *reinterpret_cast<uint4*>(orow + cc + x) = v;
            }
          }
        }
      }
    } else if (n == 0 && valid) {
      __nv_bfloat16* orow = O + (bh * N + qrow) * static_cast<long long>(D);
      for (int x = 0; x < D; x += 8) *reinterpret_cast<uint4*>(orow + x) = make_uint4(0u, 0u, 0u, 0u);
    }
    if (threadIdx.x == 128 && stats) {
      atomicAdd(&stats[0], kept_pairs);
      atomicAdd(&stats[1], skipped_pairs);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

}  // namespace sa
