// Stage 2 kernel: block-sparse attention forward on sm_100a (tcgen05 + TMA + TMEM),
// with the online-softmax-aware P.V skip.
//
// Stage 2 of the SpargeAttn abstract: the attention is computed only on the kept
// blocks (stage 1 drops the matmuls of the blocks it predicts unimportant), and an
// online-softmax-aware filter skips more P.V products at no extra cost. The DynSparse article places
// the selection inside the FlashAttention operator; this kernel is that operator.
//
// One CTA = one 128-row query tile = two 64-row query blocks (qa, qb) of one head,
// paired by the plan so that their kept sets overlap (natural pairs (2t, 2t+1)
// without a plan order). The tile walks the ascending union of the two blocks'
// kept key blocks; the half that did not keep a block sees it fully masked, so
// each 64-row query block gets exactly its own mask. Per key block j (64 keys):
//   S = Q K_j^T     128x64 fp32 into TMEM (tcgen05.mma, Q and K_j TMA'd into
//                   128B-swizzled shared memory, both K-major)
//   softmax warps   read S from TMEM (thread = row), row max, lambda vote per
//                   64-row half, exp2, row sum; P (bf16) written to TMEM
//   O += P V_j      128xD fp32 in TMEM; A operand (P) read from TMEM, B (V_j)
//                   from shared memory as an MN-major operand
//
// Roles (192 threads): warp 0 builds the union list, then one of its threads
// loads V and issues the P.V MMAs; warp 1 owns TMEM and one of its threads loads
// Q (at once, while the list is built) and K and issues the S MMAs (TMA, K and V as one 4-D box per 64-row block,
// since TMA issue cost is per instruction); warps 2..5 run the softmax (thread =
// row; warp w reaches TMEM lanes 32*(w%4) .. 32*(w%4)+31), the O correction and
// the epilogue. The issue of a tcgen05.mma that accumulates into the result of
// the previous one waits for it, so S and P.V get a thread each: S(k+1) is issued
// as soon as S(k) is released, whatever P(k-1).V is doing.
//
// TMEM (256 columns): S [0,64), P double buffer [64,96) and [96,128), O [128,
// 128+D). S is released as soon as the softmax warps hold S(k) in registers, so
// S(k+1) runs on the tensor cores while the softmax works on S(k); P(k) goes to
// buffer k&1 once its previous reader, P(k-2).V, has finished (a wait that has
// normally long passed). Two CTAs fit on an SM
// (about 106 KB of shared memory and 256 TMEM columns each), so one CTA's softmax
// also overlaps the other's MMAs.
//
// The running max used for the exponentials is raised lazily (only when a row's
// max grows by more than 2^8), which leaves O/l unchanged and makes the O
// correction rare. The lambda test uses the exact running max. Each warp posts its
// lambda vote right after the row max and reads the other warp's vote of the half
// after its exponentials, so the exchange rarely waits.
//
// An mbarrier wait by parity is only sound when the barrier is at most one phase
// ahead of, and at most one phase short of, the phase waited for; otherwise the
// parity aliases and the wait returns early or never. Every wait below satisfies
// that: S(k+1) is issued only after all softmax warps released S(k); P(k+2) is
// published only after the softmax warps have seen P(k).V finish, so the P.V
// thread has waited for P(k) by then; the P.V completions are double-buffered like
// P, and the softmax waits on them for P(k-2) (and, to correct O, P(k-1)) after
// having waited for P(k-4) (P(k-3)) before. A K or V stage is refilled only after
// the MMA that read it has completed. The lambda votes carry the
// entry index as a tag, and a vote slot is reused for entry k+2 only after every
// softmax warp has released S(k+1), which each does after reading entry k's vote
// (a warp whose own rows do not all pass cannot skip and does not read it).
// The recall filter (kRecall, below) uses the same slots, posting its vote after
// the exponentials instead; the argument is unchanged.
#pragma once

#include "sa_device.cuh"

namespace sa {

// kQ: the score operands. kScoreBF16: bf16 Q and K. kScoreE4M3 / kScoreI8: Q and
// K arrive as 8-bit codes (FP8 E4M3 or signed INT8) with one scale per 64-token
// block (d = 128 only); S = Q K^T runs as tcgen05.mma kind::f8f6f4 (fp32
// accumulate) or kind::i8 (s32 accumulate), and the two block scales join the
// softmax scale. V, P and O are as in the bf16 kernel.
template <int D, int kQ = kScoreBF16>
struct FwdCfg {
  static constexpr bool kF8 = kQ != kScoreBF16;        // 8-bit score codes
  static_assert(!kF8 || D == 128, "the 8-bit-score kernel is for d = 128");
  static constexpr int kRows = 128;                    // query rows per tile
  static constexpr int kThreads = 192;                 // 2 role warps + 4 softmax warps
  static constexpr int kChunks = D / 64;               // 128-byte (64 x bf16) column chunks of V
  static constexpr int kQKChunks = kF8 ? 1 : kChunks;  // 128-byte column chunks of a Q or K row
  static constexpr int STK = (D == 64 || kF8) ? 4 : 2; // K ring stages
  static constexpr int STV = (D == 64) ? 4 : 2;        // V ring stages
  static constexpr int kQChunkBytes = kRows * 128;     // 16 KB
  static constexpr int kKVChunkBytes = kBlock * 128;   // 8 KB
  static constexpr int kQBytes = kQKChunks * kQChunkBytes;
  static constexpr int kKBytes = kQKChunks * kKVChunkBytes;   // one K stage (also one query block of Q)
  static constexpr int kKVBytes = kChunks * kKVChunkBytes;    // one V stage
  static constexpr int kSSteps = kF8 ? D / 32 : D / 16;       // K-steps of one S MMA group
  // shared-memory layout (offsets from a 1024-aligned base)
  static constexpr int oQ = 0;
  static constexpr int oK = oQ + kQBytes;
  static constexpr int oV = oK + STK * kKBytes;
  static constexpr int oBar = oV + STV * kKVBytes;     // mbarriers
  static constexpr int kNumBars = 2 * STK + 2 * STV + 8;
  static constexpr int oMisc = oBar + kNumBars * 8;    // small words (256 bytes)
  static constexpr int oList = oMisc + 256;
  static constexpr int oListScale = oList + kMaxNb * 2;                      // kF8: K block scale per entry
  static constexpr int kSmemBytes = oListScale + (kF8 ? kMaxNb * 4 : 0) + 1024;  // + alignment slack
  // TMEM columns: S, two P buffers (bf16 pairs), the O accumulator
  static constexpr uint32_t kColS = 0, kColP0 = 64, kColP1 = 96, kColO = 128;
  static constexpr uint32_t kTmemCols = 256;
  static constexpr uint32_t kIdescS = kQ == kScoreI8 ? idesc_s8_s32(128, 64)
                                      : (kF8 ? idesc_e4m3_f32(128, 64) : idesc_bf16_f32(128, 64, false));
  static constexpr uint32_t kIdescPV = idesc_bf16_f32(128, D, true);
};

// Union-list entry: key block index (12 bits) and one keep bit per 64-row half.
constexpr uint32_t kListJMask = 0x0FFFu;
constexpr uint32_t kListLo = 1u << 14, kListHi = 1u << 15;

// p = 2^(s * scale_log2 - mref) for the 64 columns of one row; P as bf16 pairs
// and the fp32 sum of the p. Scale-subtract and sums on fp32 pairs.
__device__ __forceinline__ float softmax_exp64(const float (&s)[64], float scale_log2, float mref,
                                               uint32_t (&pk)[32]) {
  const uint64_t sc2 = f2pack(scale_log2, scale_log2), nm2 = f2pack(-mref, -mref);
  uint64_t acc0 = f2pack(0.f, 0.f), acc1 = acc0;
#pragma unroll
  for (int c = 0; c < 64; c += 2) {
    float x0, x1;
    f2unpack(ffma2(f2pack(s[c], s[c + 1]), sc2, nm2), x0, x1);
    const float p0 = ex2(x0), p1 = ex2(x1);
    if ((c >> 1) & 1)
      acc1 = fadd2(acc1, f2pack(p0, p1));
    else
      acc0 = fadd2(acc0, f2pack(p0, p1));
    pk[c >> 1] = pack_bf16x2(p0, p1);
  }
  float r0, r1, r2, r3;
  f2unpack(acc0, r0, r1);
  f2unpack(acc1, r2, r3);
  return (r0 + r1) + (r2 + r3);
}

// kRecall: the P.V filter is the cumulative-energy (recall) test instead of the
// lambda test. Each row keeps, beside its running sum l (the energy of the keys
// it has seen, relative to the reference max), the part sk of l whose P.V was
// skipped. A half skips P.V of entry k when each of its rows that sees a key of
// the block has sk*alpha + e <= budget * (l*alpha + e), e = the row's sum of P(k)
// and budget = 1 - recall; then sk takes e. So sk <= budget * l throughout and
// every row keeps at least the fraction `recall` of the energy it has seen. The
// vote needs e, so it is posted after the exponentials; the exchange is the
// lambda vote's.
// decisions (optional, [B,H,Nb,Nb] bytes): for every (query block, kept key
// block) pair the tile visits, 1 if the filter skipped its P.V, else 0.
template <int D, int kQ, bool kRecall = false>
__global__ void __launch_bounds__(192, 2)
    fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const uint8_t* __restrict__ mask,
               const int* __restrict__ work, __nv_bfloat16* __restrict__ O, int N, int Nb, int Tq,
               long long num_tiles, long long num_qblocks, float scale_log2, float lam_log2, int lam_on,
               float budget, int causal, unsigned long long* __restrict__ stats,
               const float* __restrict__ qscale, const float* __restrict__ kscale,
               uint8_t* __restrict__ decisions) {
  using C = FwdCfg<D, kQ>;
  constexpr bool kF8 = C::kF8;                   // 8-bit score codes (E4M3 or INT8)
  constexpr bool kI8 = kQ == kScoreI8;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = base + C::oQ;
  uint8_t* sK = base + C::oK;
  uint8_t* sV = base + C::oV;
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + C::oBar);
  uint64_t* kfull = bars;                      // [STK] K stage loaded
  uint64_t* kempty = kfull + C::STK;           // [STK] K stage consumed by S MMA
  uint64_t* vfull = kempty + C::STK;           // [STV] V stage loaded
  uint64_t* vempty = vfull + C::STV;           // [STV] V stage consumed by P.V MMA
  uint64_t* q_full = vempty + C::STV;          // Q tile loaded
  uint64_t* s_full = q_full + 1;               // S(k) written by the MMA (phase k)
  uint64_t* s_free = q_full + 2;               // S(k) read by all 4 softmax warps (phase k)
  uint64_t* p_full = q_full + 3;               // [2] by k parity: P(k) in TMEM and O corrected (4 warps)
  uint64_t* pv_done = q_full + 5;              // [2] by k parity: P(k).V finished
  uint64_t* drain = q_full + 7;                // every MMA of the tile finished (single phase, 2 issuers)
  int* misc = reinterpret_cast<int*>(base + C::oMisc);
  volatile int* abort_flag = misc + 0;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(misc + 1);
  int* list_n = misc + 2;
  volatile int* contrib = misc + 4;            // [2 parity][2 halves]: the half's P.V is needed
  volatile int* votes = misc + 8;              // [2 parity][4 softmax warps]: (k << 1) | pass
  uint16_t* lst = reinterpret_cast<uint16_t*>(base + C::oList);
  float* lsk = reinterpret_cast<float*>(base + C::oListScale);   // kF8: K block scale of each entry

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (blockIdx.x >= num_tiles) return;
  long long ga, gb;  // global query-block ids (b*H + h)*Nb + i of the two halves
  if (work) {
    ga = work[2 * static_cast<long long>(blockIdx.x)];
    gb = work[2 * static_cast<long long>(blockIdx.x) + 1];
  } else {
    const long long bh0 = blockIdx.x / Tq;
    const int t = static_cast<int>(blockIdx.x - bh0 * Tq);
    ga = bh0 * Nb + 2 * t;
    gb = (2 * t + 1 < Nb) ? ga + 1 : -1;
  }
  if (ga < 0 || ga >= num_qblocks || gb < -1 || gb >= num_qblocks || (gb >= 0 && gb / Nb != ga / Nb)) {
    if (threadIdx.x == 0) atomicOr(&g_dev_error, DEVERR_RANGE);  // corrupt work list: skip
    return;
  }
  const long long bh = ga / Nb;
  const int qb0 = static_cast<int>(ga - bh * Nb);              // query block of rows 0..63
  const int qb1 = gb >= 0 ? static_cast<int>(gb - bh * Nb) : -1;  // rows 64..127 (-1: none)

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STK; ++s) {
      mbar_init(&kfull[s], 1);
      mbar_init(&kempty[s], 1);
    }
    for (int s = 0; s < C::STV; ++s) {
      mbar_init(&vfull[s], 1);
      mbar_init(&vempty[s], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(s_free, 4);
    mbar_init(&p_full[0], 4);
    mbar_init(&p_full[1], 4);
    mbar_init(&pv_done[0], 1);
    mbar_init(&pv_done[1], 1);
    mbar_init(drain, 2);
    *abort_flag = 0;
    for (int x = 8; x < 16; ++x) misc[x] = -1;   // vote tags -1: no entry yet
    fence_mbar_init();
  }
  if (warp == 1) {
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      // Q rows of the two query blocks into rows 0..63 / 64..127 of the tile, issued
      // now so that the load overlaps warp 0's build of the union list
      mbar_init(q_full, 1);
      fence_mbar_init();
      mbar_expect_tx(q_full, (qb1 >= 0 ? 2 : 1) * C::kKBytes);
#pragma unroll
      for (int c = 0; c < C::kQKChunks; ++c) {
        tma_load_3d(sQ + c * C::kQChunkBytes, &tmQ, c * 64, qb0 * kBlock, static_cast<int>(bh), q_full);
        if (qb1 >= 0)
          tma_load_3d(sQ + c * C::kQChunkBytes + C::kKVChunkBytes, &tmQ, c * 64, qb1 * kBlock,
                      static_cast<int>(bh), q_full);
      }
    }
    __syncwarp();
    tmem_alloc(tmem_holder, C::kTmemCols);
  }
  if (warp == 0) {
    // Ascending union of the kept lists of query blocks qb0 and qb1, one keep bit
    // per half; with causal, key blocks after a half's query block are dropped.
    const uint8_t* m0 = mask + (bh * Nb + qb0) * static_cast<long long>(Nb);
    const uint8_t* m1 = (qb1 >= 0) ? mask + (bh * Nb + qb1) * static_cast<long long>(Nb) : nullptr;
    const int jend = causal ? min(Nb, max(qb0, qb1) + 1) : Nb;
    int n = 0;
    for (int jb = 0; jb < jend; jb += 128) {
      uint32_t a[4], b[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {  // independent loads first
        const int j = jb + 32 * u + lane;
        a[u] = (j < jend) ? static_cast<uint32_t>(m0[j] != 0) : 0u;
        b[u] = (j < jend && m1 != nullptr) ? static_cast<uint32_t>(m1[j] != 0) : 0u;
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int j = jb + 32 * u + lane;
        if (causal) {
          a[u] &= (j <= qb0) ? 1u : 0u;
          b[u] &= (j <= qb1) ? 1u : 0u;
        }
        const uint32_t any = a[u] | b[u];
        const unsigned bal = __ballot_sync(0xffffffffu, any != 0);
        if (any)
          lst[n + __popc(bal & ((1u << lane) - 1u))] =
              static_cast<uint16_t>(static_cast<uint32_t>(j) | (a[u] ? kListLo : 0u) | (b[u] ? kListHi : 0u));
        n += __popc(bal);
      }
    }
    if (lane == 0) *list_n = n;
    if constexpr (kF8) {
      __syncwarp();
      for (int e = lane; e < n; e += 32) lsk[e] = kscale[bh * Nb + (lst[e] & kListJMask)];
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const int n = *list_n;

  if (warp == 0) {
    // ------------------------------------------------------------ V producer, P.V issuer
    if (lane == 0 && n > 0) {
      const uint32_t sVa = smem_u32(sV);
      auto load_v = [&](int k) {
        const int s = k % C::STV;
        const int j = static_cast<int>(lst[k] & kListJMask);
        mbar_expect_tx(&vfull[s], C::kKVBytes);
        tma_load_4d(sV + s * C::kKVBytes, &tmV, 0, j * kBlock, 0, static_cast<int>(bh), &vfull[s]);
      };
      int nv = 0;                                 // V loads issued
      for (; nv < C::STV && nv < n; ++nv) load_v(nv);
      uint32_t o_init = 0;
      unsigned long long pv_tiles = 0;
      for (int k = 0; k < n; ++k) {
        if (!mbar_wait(&p_full[k & 1], static_cast<uint32_t>(k >> 1) & 1u, abort_flag)) break;
        const int s = k % C::STV;
        if (!mbar_wait(&vfull[s], static_cast<uint32_t>(k / C::STV) & 1u, abort_flag)) break;
        tc_fence_after();
        if (contrib[(k & 1) * 2] | contrib[(k & 1) * 2 + 1]) {
          const uint32_t dO = tmem_base + C::kColO;
          const uint32_t aP = tmem_base + ((k & 1) ? C::kColP1 : C::kColP0);
#pragma unroll
          for (int kk = 0; kk < kBlock / 16; ++kk) {
            const uint64_t bd = sdesc_sw128(sVa + s * C::kKVBytes + kk * 16 * 128, C::kKVChunkBytes, 1024);
            tc_mma_ts(dO, aP + kk * 8, bd, C::kIdescPV, (o_init | static_cast<uint32_t>(kk > 0)));
          }
          o_init = 1u;
          ++pv_tiles;
        }
        tc_commit(&pv_done[k & 1]);
        tc_commit(&vempty[s]);
        // refill this stage with V(k+STV) once P(k).V has read it
        if (k + C::STV < n) {
          if (!mbar_wait(&vempty[s], static_cast<uint32_t>(k / C::STV) & 1u, abort_flag)) break;
          load_v(k + C::STV);
          ++nv;
        }
      }
      // Drain: every MMA this thread issued has finished and its loads have landed
      // (bounded); the softmax warps wait on the same barrier before reading O.
      tc_commit(drain);
      mbar_wait_drain(drain, 0u);
      for (int kk = max(0, nv - C::STV); kk < nv; ++kk)
        mbar_wait_drain(&vfull[kk % C::STV], static_cast<uint32_t>(kk / C::STV) & 1u);
      if (stats) atomicAdd(&stats[3], pv_tiles);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ Q, K producer, S issuer
    if (lane == 0 && n > 0) {
      auto load_k = [&](int k) {
        const int s = k % C::STK;
        const int j = static_cast<int>(lst[k] & kListJMask);
        mbar_expect_tx(&kfull[s], C::kKBytes);
        if constexpr (kF8)
          tma_load_3d(sK + s * C::kKBytes, &tmK, 0, j * kBlock, static_cast<int>(bh), &kfull[s]);
        else
          tma_load_4d(sK + s * C::kKBytes, &tmK, 0, j * kBlock, 0, static_cast<int>(bh), &kfull[s]);
      };
      int nk = 0;                                 // K loads issued
      for (; nk < C::STK && nk < n; ++nk) load_k(nk);
      const uint32_t sQa = smem_u32(sQ), sKa = smem_u32(sK);
      bool ok = mbar_wait(q_full, 0u, abort_flag);
      // S(k) = Q K_k^T into the S columns, once the softmax warps released S(k-1)
      for (int k = 0; ok && k < n; ++k) {
        if (k > 0 && !mbar_wait(s_free, static_cast<uint32_t>(k - 1) & 1u, abort_flag)) break;
        const int s = k % C::STK;
        if (!mbar_wait(&kfull[s], static_cast<uint32_t>(k / C::STK) & 1u, abort_flag)) break;
        tc_fence_after();
        const uint32_t dS = tmem_base + C::kColS;
#pragma unroll
        for (int kk = 0; kk < C::kSSteps; ++kk) {
          const uint32_t off = (kk & 3) * 32;  // 16 bf16 or 32 e4m3 = 32 bytes inside the swizzle atom
          const uint64_t ad = sdesc_sw128(sQa + (kk >> 2) * C::kQChunkBytes + off, 16, 1024);
          const uint64_t bd = sdesc_sw128(sKa + s * C::kKBytes + (kk >> 2) * C::kKVChunkBytes + off, 16, 1024);
          if constexpr (kI8)
            tc_mma_ss_i8(dS, ad, bd, C::kIdescS, kk > 0 ? 1u : 0u);
          else if constexpr (kF8)
            tc_mma_ss_f8(dS, ad, bd, C::kIdescS, kk > 0 ? 1u : 0u);
          else
            tc_mma_ss(dS, ad, bd, C::kIdescS, kk > 0 ? 1u : 0u);
        }
        tc_commit(s_full);
        tc_commit(&kempty[s]);
        // refill this stage with K(k+STK) once S(k) has read it
        if (k + C::STK < n) {
          if (!mbar_wait(&kempty[s], static_cast<uint32_t>(k / C::STK) & 1u, abort_flag)) break;
          load_k(k + C::STK);
          ++nk;
        }
      }
      tc_commit(drain);
      mbar_wait_drain(drain, 0u);
      mbar_wait_drain(q_full, 0u);
      for (int kk = max(0, nk - C::STK); kk < nk; ++kk)
        mbar_wait_drain(&kfull[kk % C::STK], static_cast<uint32_t>(kk / C::STK) & 1u);
      if (stats) atomicAdd(&stats[2], static_cast<unsigned long long>(n));
    } else if (lane == 0) {
      mbar_wait_drain(q_full, 0u);                // no entry: the Q load still lands first
    }
  } else if (warp >= 2) {
    // ------------------------------------------------------------ softmax warps
    const int wq = warp & 3;                     // TMEM lane quadrant: rows 32*wq .. 32*wq+31
    const int row = wq * 32 + lane;              // tile row == TMEM lane
    const int half = wq >> 1;                    // quadrants 0,1 -> query block qb0; 2,3 -> qb1
    const int myqb = half ? qb1 : qb0;
    const long long qrow = static_cast<long long>(myqb) * kBlock + (row & (kBlock - 1));
    const bool valid = myqb >= 0 && qrow < N;
    const uint32_t lane_bits = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t s_addr = tmem_base + lane_bits + C::kColS;
    const uint32_t o_addr = tmem_base + lane_bits + C::kColO;
    const bool writer = (wq & 1) == 0 && lane == 0;   // one per half: contrib, stats
    // kF8: the scores are codes; this row's query-block scale joins the softmax scale
    const float sqh = kF8 ? (myqb >= 0 ? qscale[bh * Nb + myqb] : 1.f) : 1.f;
    const unsigned FULL = 0xffffffffu;
    float m_true = -INFINITY, m_ref = -INFINITY, l = 0.f;
    float sk = 0.f;                              // kRecall: skipped part of l
    unsigned long long kept_pairs = 0, skipped_pairs = 0;
    bool alive = true;
    // S(k) is loaded from TMEM one entry ahead: the load of S(k+1) is issued while
    // the store of P(k) is still in flight.
    float s[64];
    if (n > 0) {
      if (warp_wait(s_full, 0u, abort_flag)) {
        tc_fence_after();
        tmem_ld32(s_addr, *reinterpret_cast<float(*)[32]>(&s[0]));
        tmem_ld32(s_addr + 32, *reinterpret_cast<float(*)[32]>(&s[32]));
      } else {
        alive = false;
      }
    }
    for (int k = 0; alive && k < n; ++k) {
      const uint32_t e = lst[k];
      const int j = static_cast<int>(e & kListJMask);
      const bool keep_lo = (e & kListLo) != 0u, keep_hi = (e & kListHi) != 0u;
      const bool keep = half ? keep_hi : keep_lo;
      const int kbase = j * kBlock;
      // visible columns of this row in the block: c < ncol (tail, causal diagonal)
      int ncol = (keep && valid) ? min(kBlock, N - kbase) : 0;
      if (causal) ncol = min(ncol, static_cast<int>(max(qrow - kbase + 1, 0LL)));
      const bool warp_none = __all_sync(FULL, ncol == 0);
      const bool warp_full = __all_sync(FULL, ncol == kBlock);
      const float sc = kF8 ? scale_log2 * sqh * lsk[k] : scale_log2;   // log2-domain scale of S(k)
      tmem_wait_ld();                             // S(k) is in s[]
      pin32(*reinterpret_cast<float(*)[32]>(&s[0]));
      pin32(*reinterpret_cast<float(*)[32]>(&s[32]));
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(s_free);         // S may now be overwritten by S(k+1)
      if constexpr (kI8) {
        // s32 scores (|S| < 2^22) to the exact floats 12582912 + S: the integer
        // plus the bits of 1.5 * 2^23 (ordered like S); the offset is taken out
        // of the row max below and folded into the exponentials' bias
#pragma unroll
        for (int c = 0; c < 64; ++c) s[c] = __int_as_float(__float_as_int(s[c]) + 0x4B400000);
      }
      uint32_t pk[32];                            // P as packed bf16 pairs
      float rmax = -INFINITY, psum = 0.f;
      if (!warp_none) {
        if (!warp_full) {
#pragma unroll
          for (int c = 0; c < 64; ++c) s[c] = (c < ncol) ? s[c] : -INFINITY;
        }
        float mx[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) mx[u] = fmax3(s[u], s[u + 8], s[u + 16]);
#pragma unroll
        for (int c = 24; c < 56; c += 16) {
#pragma unroll
          for (int u = 0; u < 8; ++u) mx[u] = fmax3(mx[u], s[c + u], s[c + 8 + u]);
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) mx[u] = fmaxf(mx[u], s[56 + u]);
        float mxv = fmax3(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7]));
        if constexpr (kI8) mxv -= 12582912.f;    // exact: back to the integer score
        rmax = mxv * sc;                          // -inf stays -inf (sc > 0)
      }
      bool wpass = true;
      if (!kRecall && lam_on) {
        // this warp's lambda vote, posted before the exponentials so that the other
        // warp of the half finds it when it needs it
        const bool pass = !(rmax > -INFINITY) || (rmax - m_true < lam_log2);
        wpass = __all_sync(FULL, pass);
        if (lane == 0) votes[(k & 1) * 4 + wq] = (k << 1) | (wpass ? 1 : 0);
      }
      const float m_new = fmaxf(m_true, rmax);
      const bool raise = m_new > m_ref + 8.f;    // also true for the first finite max
      float alpha = 1.f;
      if (raise) {
        alpha = ex2(m_ref - m_new);               // 0 when m_ref = -inf
        m_ref = m_new;
      }
      const bool any_raise = __any_sync(FULL, raise);
      float mref = (m_ref == -INFINITY) ? 0.f : m_ref;
      asm volatile("" : "+f"(mref) :: "memory");  // the exponentials after the vote is posted
      if (warp_none) {
#pragma unroll
        for (int c = 0; c < 32; ++c) pk[c] = 0u;
      } else {
        // INT8: s holds 12582912 + S, so the bias also takes 12582912 * sc
        psum = softmax_exp64(s, sc, kI8 ? mref + 12582912.f * sc : mref, pk);
      }
      m_true = m_new;
      l = l * alpha + psum;
      float sk_try = 0.f;
      if (kRecall) {
        // this warp's recall vote (rows that see no key of the block have no say)
        sk_try = sk * alpha + psum;
        const bool pass = ncol == 0 || sk_try <= budget * l;
        wpass = __all_sync(FULL, pass);
        if (lane == 0) votes[(k & 1) * 4 + wq] = (k << 1) | (wpass ? 1 : 0);
      }
      // the half skips P.V when both of its warps pass; its P(k) is zero
      bool half_skip = false;
      if (lam_on && wpass) {                      // a warp that does not pass never skips
        int pv = 0;
        if (lane == 0) pv = spin_tag(&votes[(k & 1) * 4 + (wq ^ 1)], k, abort_flag);
        pv = __shfl_sync(FULL, pv, 0);
        if (pv < 0) { alive = false; break; }
        half_skip = (pv & 1) != 0;
        if (half_skip) {
#pragma unroll
          for (int c = 0; c < 32; ++c) pk[c] = 0u;
        }
      }
      if (kRecall) sk = half_skip ? sk_try : sk * alpha;
      // P(k) into buffer k&1 once its previous reader, P(k-2).V, has finished
      if (k >= 2) {
        if (!warp_wait(&pv_done[k & 1], static_cast<uint32_t>((k - 2) >> 1) & 1u, abort_flag)) {
          alive = false;
          break;
        }
        tc_fence_after();
      }
      tmem_st32u(tmem_base + lane_bits + ((k & 1) ? C::kColP1 : C::kColP0), pk);
      // O correction for rows whose reference max was raised (after P(k-1).V);
      // pv_done[(k-1)&1] is at most one phase short of entry k-1 (this warp waited
      // for P(k-3).V before storing P(k-1)).
      if (k > 0 && any_raise) {
        if (!warp_wait(&pv_done[(k - 1) & 1], static_cast<uint32_t>((k - 1) >> 1) & 1u, abort_flag)) {
          alive = false;
          break;
        }
        tc_fence_after();
#pragma unroll 1
        for (int cc = 0; cc < D; cc += 32) {
          float o[32];
          tmem_ld32(o_addr + cc, o);
          tmem_wait_ld();
          pin32(o);
#pragma unroll
          for (int x = 0; x < 32; ++x) o[x] *= alpha;
          tmem_st32(o_addr + cc, o);
        }
      }
      // prefetch S(k+1) while P(k) is being stored
      if (k + 1 < n) {
        if (!warp_wait(s_full, static_cast<uint32_t>(k + 1) & 1u, abort_flag)) {
          alive = false;
          break;
        }
        tc_fence_after();
        tmem_ld32(s_addr, *reinterpret_cast<float(*)[32]>(&s[0]));
        tmem_ld32(s_addr + 32, *reinterpret_cast<float(*)[32]>(&s[32]));
      }
      tmem_wait_st();
      if (writer) {
        contrib[(k & 1) * 2 + half] = (keep && !half_skip) ? 1 : 0;
        kept_pairs += keep ? 1ull : 0ull;
        skipped_pairs += (keep && half_skip) ? 1ull : 0ull;
        if (decisions && keep) decisions[(bh * Nb + myqb) * static_cast<long long>(Nb) + j] = half_skip ? 1 : 0;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[k & 1]);
    }
    tmem_wait_ld();                               // no TMEM load left in flight
    // ------------------------------------------------------------ epilogue
    if (alive && n > 0) {
      if (warp_wait(drain, 0u, abort_flag)) {
        tc_fence_after();
        const float inv = (l > 0.f) ? 1.f / l : 0.f;
        __nv_bfloat16* orow = O + (bh * N + qrow) * static_cast<long long>(D);
#pragma unroll
        for (int cc = 0; cc < D; cc += 32) {
          float o[32];
          tmem_ld32(o_addr + cc, o);
          tmem_wait_ld();
          pin32(o);
          if (valid) {
#pragma unroll
            for (int x = 0; x < 32; x += 8) {
              uint4 v;
              v.x = pack_bf16x2(o[x + 0] * inv, o[x + 1] * inv);
              v.y = pack_bf16x2(o[x + 2] * inv, o[x + 3] * inv);
              v.z = pack_bf16x2(o[x + 4] * inv, o[x + 5] * inv);
              v.w = pack_bf16x2(o[x + 6] * inv, o[x + 7] * inv);
              *reinterpret_cast<uint4*>(orow + cc + x) = v;
            }
          }
        }
      }
    } else if (n == 0 && valid) {
      __nv_bfloat16* orow = O + (bh * N + qrow) * static_cast<long long>(D);
      for (int x = 0; x < D; x += 8) *reinterpret_cast<uint4*>(orow + x) = make_uint4(0u, 0u, 0u, 0u);
    }
    if (writer && stats) {
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
