// attn_tc.cu -- block-sparse flash attention on the 5th-generation tensor
// cores ("XAttention: Block Sparse Attention with Antidiagonal Scoring",
// §1 step 3 Block Sparse Attention: attention computed over the selected
// blocks only).
//
// A work unit is one (batch*head, query block) with its ascending list of key
// blocks (B = 128, d = 128). For each listed key block j:
//   S_j = Q K_j^T                 tcgen05.mma, A = Q (smem), B = K_j (smem) -> TMEM
//   P_j = exp2(S_j * c - m)       softmax warps, one TMEM lane (query row) each,
//                                 online max with lazy rescaling of O
//   O  += P_j V_j                 tcgen05.mma, A = P_j (TMEM, bf16), B = V_j (smem)
// P_j is written back over the first 64 TMEM columns of S_j as packed bf16, so
// a CTA needs 256 TMEM columns (S 128 + O 128). Two CTAs share an SM, and
// the tensor core switches between them: one CTA's softmax overlaps the
// other's MMAs.
//
// Warp roles (192 threads):
//   warp 0      TMA producer: Q once per unit, then K_j, V_j into a 2-slot ring
//   warp 1      TMEM allocator + MMA issuer
//   warps 2..5  softmax and output epilogue (warp w owns TMEM lanes 32*(w%4)..)
// Units come from the longest-list-first order, round-robin over the CTAs.
// Every pipeline wait is bounded; on time-out the CTA raises its abort flag,
// drains, frees TMEM and records XATTN_ERR_TIMEOUT in the status word.
#include <cuda_bf16.h>

#include "common.cuh"
#include "ptx.cuh"

namespace xattn {
namespace {

constexpr int kThreads = 192;
constexpr int kBlk = 128;                      // B (rows per query / key block)
constexpr int kD = 128;                        // head dim
constexpr int kHalf = kBlk * 64 * 2;           // one 64-feature box: 16 KB
constexpr int kTileBytes = 2 * kHalf;          // 128 x 128 bf16: 32 KB
constexpr int kStages = 2;
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kColS = 0;                  // S_j (fp32), P_j (bf16) aliases cols 0..63
constexpr uint32_t kColO = 128;                // O accumulator (fp32)
constexpr uint32_t kIdescS = idesc_bf16_f32(kBlk, kBlk, 0, 0);
constexpr uint32_t kIdescPV = idesc_bf16_f32(kBlk, kD, 0, 1);  // V is MN-major
constexpr float kRescaleLog2 = 8.0f;           // rescale O only when the max grows by > 2^8

struct Params {
  int L, NB, hq, hkv, group, causal, units;
  float scale_log2;  // log2(e) / sqrt(d)
  const int32_t* counts;
  const int32_t* idx;
  const uint32_t* order;
  __nv_bfloat16* O;
  float* lse;
  int* status;
};

struct Smem {
  uint64_t q_full, q_empty;
  uint64_t kv_full[kStages], kv_empty[kStages];
  uint64_t s_full, p_full, pv_done, o_empty;
  uint32_t tmem_base;
  int abort;
};

// Number of listed blocks a unit actually uses: causal lists drop the
// trailing blocks above the diagonal (the list is ascending).
__device__ __forceinline__ int effective_count(const Params& p, const int32_t* list, int n,
                                               int qb) {
  n = n < 0 ? 0 : (n > p.NB ? p.NB : n);
  if (!p.causal) return n;
  while (n > 0 && list[n - 1] > qb) --n;
  return n;
}

__global__ void __launch_bounds__(kThreads, 2)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ,
                   const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* q_smem = base;
  uint8_t* kv_smem = base + kTileBytes;
  Smem* sm = reinterpret_cast<Smem*>(base + kTileBytes * (1 + kStages));

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    mbar_init(&sm->q_full, 1);
    mbar_init(&sm->q_empty, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm->kv_full[s], 1);
      mbar_init(&sm->kv_empty[s], 1);
    }
    mbar_init(&sm->s_full, 1);
    mbar_init(&sm->p_full, 128);
    mbar_init(&sm->pv_done, 1);
    mbar_init(&sm->o_empty, 128);
    sm->abort = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  if (warp == 1) {
    tmem_alloc(&sm->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm->tmem_base;
  volatile int* abort = &sm->abort;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------ TMA producer
      int stage = 0;
      uint32_t phase = 0;
      uint32_t nu = 0;  // units with work seen so far
      long long issued = 0;
      bool q_out = false;
      for (int k = blockIdx.x; k < p.units && !*abort; k += gridDim.x) {
        const int unit = static_cast<int>(p.order[k]);
        const int bh = unit / p.NB, qb = unit % p.NB;
        const int32_t* list = p.idx + static_cast<size_t>(unit) * p.NB;
        const int n = effective_count(p, list, p.counts[unit], qb);
        if (n <= 0) continue;
        const int kvbh = (bh / p.hq) * p.hkv + (bh % p.hq) / p.group;
        if (!mbar_wait(&sm->q_empty, (nu & 1) ^ 1, abort)) break;
        mbar_arrive_expect_tx(&sm->q_full, kTileBytes);
        const int qrow = bh * p.L + qb * kBlk;
        tma_load_2d(q_smem, &tmQ, &sm->q_full, 0, qrow);
        tma_load_2d(q_smem + kHalf, &tmQ, &sm->q_full, 64, qrow);
        q_out = true;
        for (int j = 0; j < n; ++j) {
          const int krow = kvbh * p.L + list[j] * kBlk;
          for (int which = 0; which < 2; ++which) {  // K_j then V_j
            if (!mbar_wait(&sm->kv_empty[stage], phase ^ 1, abort)) goto producer_done;
            uint8_t* dst = kv_smem + stage * kTileBytes;
            const CUtensorMap* map = which == 0 ? &tmK : &tmV;
            mbar_arrive_expect_tx(&sm->kv_full[stage], kTileBytes);
            tma_load_2d(dst, map, &sm->kv_full[stage], 0, krow);
            tma_load_2d(dst + kHalf, map, &sm->kv_full[stage], 64, krow);
            ++issued;
            if (++stage == kStages) {
              stage = 0;
              phase ^= 1;
            }
          }
        }
        ++nu;
      }
    producer_done:
      if (*abort) {
        // wait (bounded) for the copies this thread still has in flight
        const long long nk = issued < kStages ? issued : kStages;
        for (long long t = 1; t <= nk; ++t) {
          const long long q = issued - t;
          const uint32_t addr = smem_u32(&sm->kv_full[q % kStages]);
          const uint32_t ph = static_cast<uint32_t>((q / kStages) & 1);
          const unsigned long long t0 = globaltimer();
          while (!mbar_try_wait(addr, ph) && globaltimer() - t0 < kWaitLimitNs) {
          }
        }
        if (q_out && nu > 0) {
          const uint32_t addr = smem_u32(&sm->q_full);
          const unsigned long long t0 = globaltimer();
          while (!mbar_try_wait(addr, (nu - 1) & 1) && globaltimer() - t0 < kWaitLimitNs) {
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------ MMA issuer
      int stage = 0;
      uint32_t phase = 0;
      uint32_t nu = 0;
      uint32_t g = 0;  // global block counter of this CTA
      const uint32_t q_addr = smem_u32(q_smem);
      for (int k = blockIdx.x; k < p.units; k += gridDim.x) {
        const int unit = static_cast<int>(p.order[k]);
        const int qb = unit % p.NB;
        const int32_t* list = p.idx + static_cast<size_t>(unit) * p.NB;
        const int n = effective_count(p, list, p.counts[unit], qb);
        if (n <= 0) continue;
        if (!mbar_wait(&sm->q_full, nu & 1, abort)) goto mma_done;
        for (int j = 0; j < n; ++j, ++g) {
          // S_j = Q K_j^T
          if (!mbar_wait(&sm->kv_full[stage], phase, abort)) goto mma_done;
          tc_fence_after();
          {
            const uint32_t k_addr = smem_u32(kv_smem + stage * kTileBytes);
#pragma unroll
            for (int kk = 0; kk < kD / 16; ++kk) {
              const uint32_t off = (kk >> 2) * kHalf + (kk & 3) * 32;
              umma_ss(tmem + kColS, smem_desc_sw128(q_addr + off, 16, 1024),
                      smem_desc_sw128(k_addr + off, 16, 1024), kIdescS, kk > 0);
            }
          }
          umma_commit(&sm->s_full);
          umma_commit(&sm->kv_empty[stage]);
          if (j == n - 1) umma_commit(&sm->q_empty);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1;
          }
          // O += P_j V_j
          if (!mbar_wait(&sm->p_full, g & 1, abort)) goto mma_done;
          if (j == 0 && !mbar_wait(&sm->o_empty, (nu & 1) ^ 1, abort)) goto mma_done;
          if (!mbar_wait(&sm->kv_full[stage], phase, abort)) goto mma_done;
          tc_fence_after();
          {
            const uint32_t v_addr = smem_u32(kv_smem + stage * kTileBytes);
#pragma unroll
            for (int kk = 0; kk < kBlk / 16; ++kk) {
              // 16 keys per step: P columns [8kk, 8kk+8) (bf16 pairs), V rows [16kk, 16kk+16)
              umma_ts(tmem + kColO, tmem + kColS + kk * 8,
                      smem_desc_sw128(v_addr + kk * 16 * 128, kHalf, 1024), kIdescPV,
                      (j > 0 || kk > 0) ? 1u : 0u);
            }
          }
          umma_commit(&sm->pv_done);
          umma_commit(&sm->kv_empty[stage]);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1;
          }
        }
        ++nu;
      }
    mma_done:;
    }
  } else {
    // ------------------------------------------------ softmax + epilogue
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tS = tmem + lane_addr + kColS;
    const uint32_t tO = tmem + lane_addr + kColO;
    const float sl2 = p.scale_log2;
    uint32_t g = 0;
    for (int k = blockIdx.x; k < p.units; k += gridDim.x) {
      const int unit = static_cast<int>(p.order[k]);
      const int bh = unit / p.NB, qb = unit % p.NB;
      const int32_t* list = p.idx + static_cast<size_t>(unit) * p.NB;
      const int n = effective_count(p, list, p.counts[unit], qb);
      const size_t orow = static_cast<size_t>(bh) * p.L + static_cast<size_t>(qb) * kBlk + row;
      __nv_bfloat16* optr = p.O + orow * kD;
      if (n <= 0) {
        uint4 z = make_uint4(0, 0, 0, 0);
        for (int c = 0; c < kD / 8; ++c) reinterpret_cast<uint4*>(optr)[c] = z;
        if (p.lse) p.lse[orow] = -INFINITY;
        continue;
      }
      float m_run = -INFINITY;  // running max of scaled logits (log2 units)
      float l_run = 0.f;
      bool failed = false;
      for (int j = 0; j < n; ++j, ++g) {
        const bool diag = p.causal && list[j] == qb;
        if (!warp_wait(&sm->s_full, g & 1, abort)) {
          failed = true;
          break;
        }
        tc_fence_after();
        float s[kBlk];
#pragma unroll
        for (int c = 0; c < kBlk / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(tS + c * 32, v);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) s[c * 32 + i] = __uint_as_float(v[i]);
        }
        if (diag) {
#pragma unroll
          for (int c = 0; c < kBlk; ++c)
            if (c > row) s[c] = -INFINITY;
        }
        float mx = -INFINITY;
#pragma unroll
        for (int c = 0; c < kBlk; ++c) mx = fmaxf(mx, s[c]);
        const float m_new = fmaxf(m_run, mx * sl2);
        const bool need = m_new > m_run + kRescaleLog2;
        if (__any_sync(0xffffffffu, need)) {
          const float alpha = need ? ex2(m_run - m_new) : 1.0f;
          if (j > 0) {
            // O holds PV_0..PV_{j-1}: wait for the last one, then rescale in place
            if (!warp_wait(&sm->pv_done, (g - 1) & 1, abort)) {
              failed = true;
              break;
            }
            tc_fence_after();
#pragma unroll 1
            for (int c = 0; c < kD / 32; ++c) {
              uint32_t v[32];
              tmem_ld32(tO + c * 32, v);
              tmem_ld_wait();
#pragma unroll
              for (int i = 0; i < 32; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) * alpha);
              tmem_st32(tO + c * 32, v);
            }
            tmem_st_wait();
          }
          if (need) {
            l_run *= alpha;
            m_run = m_new;
          }
        }
        const float mb = m_run;
        float lsum = 0.f;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          // keys [64h, 64h + 64) -> bf16 pairs in TMEM columns [32h, 32h + 32)
          uint32_t pk[32];
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const float p0 = ex2(fmaf(s[64 * h + 2 * c], sl2, -mb));
            const float p1 = ex2(fmaf(s[64 * h + 2 * c + 1], sl2, -mb));
            lsum += p0 + p1;
            pk[c] = pack_bf16x2(p0, p1);
          }
          tmem_st32(tS + 32 * h, pk);
        }
        l_run += lsum;
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&sm->p_full);
      }
      if (failed) break;
      // ---- epilogue: O / l -> bf16 rows
      if (!warp_wait(&sm->pv_done, (g - 1) & 1, abort)) break;
      tc_fence_after();
      const float inv = l_run > 0.f ? 1.0f / l_run : 0.f;
#pragma unroll 1
      for (int c = 0; c < kD / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(tO + c * 32, v);
        tmem_ld_wait();
        uint32_t w[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          w[i] = pack_bf16x2(__uint_as_float(v[2 * i]) * inv, __uint_as_float(v[2 * i + 1]) * inv);
        uint4* dst = reinterpret_cast<uint4*>(optr + c * 32);
#pragma unroll
        for (int i = 0; i < 4; ++i) dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
      }
      if (p.lse) p.lse[orow] = (m_run + lg2(l_run)) * 0.69314718055994531f;
      tc_fence_before();
      mbar_arrive(&sm->o_empty);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
  if (threadIdx.x == 0 && sm->abort) atomicExch(p.status, kStatusTimeout);
}

}  // namespace

cudaError_t launch_attn_tc(const Dims& D, const CUtensorMap& tmQ, const CUtensorMap& tmK,
                           const CUtensorMap& tmV, const int32_t* counts, const int32_t* idx,
                           const uint32_t* order, void* O, float* lse, int* status,
                           int num_sms, cudaStream_t st) {
  Params p{};
  p.L = D.L;
  p.NB = D.NB;
  p.hq = D.hq;
  p.hkv = D.hkv;
  p.group = D.group;
  p.causal = D.causal;
  p.units = D.batch * D.hq * D.NB;
  p.scale_log2 = static_cast<float>(1.4426950408889634 / sqrt(double(D.d)));
  p.counts = counts;
  p.idx = idx;
  p.order = order;
  p.O = static_cast<__nv_bfloat16*>(O);
  p.lse = lse;
  p.status = status;
  const size_t smem = 1024 + kTileBytes * (1 + kStages) + sizeof(Smem);
  cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  int grid = 2 * num_sms;
  if (grid > p.units) grid = p.units;
  if (grid < 1) grid = 1;
  attn_tc_kernel<<<grid, kThreads, smem, st>>>(tmQ, tmK, tmV, p);
  return cudaGetLastError();
}

}  // namespace xattn
