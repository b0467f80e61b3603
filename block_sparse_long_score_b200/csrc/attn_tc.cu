// attn_tc.cu -- block-sparse flash attention on the 5th-generation tensor
// cores ("XAttention: Block Sparse Attention with Antidiagonal Scoring",
// §1 step 3 Block Sparse Attention: attention computed over the selected
// blocks only).
//
// A work unit is one (batch*head, query block) with its ascending list of key
// blocks (B = 128, d = 128). For each listed key block j:
//   S_j = Q K_j^T                 tcgen05.mma, A = Q (smem), B = K_j (smem) -> TMEM
//   P_j = exp2(S_j * c - m)       softmax warps, one TMEM lane (query row) each,
//                                 running max with lazy rescaling of O
//   O  += P_j V_j                 tcgen05.mma, A = P_j (TMEM, bf16), B = V_j (smem)
// P_j is written back over the first 64 TMEM columns of S_j as packed bf16.
//
// One persistent CTA per SM runs two independent units at a time ("slots").
// Each slot has its own Q tile in shared memory, its own 256 TMEM columns
// (S 128 + O 128) and its own softmax warpgroup. One MMA thread interleaves
// the slots -- S(0), S(1), then PV(0), S(0, next), PV(1), S(1, next), ... --
// so the tensor core works on one slot while the other slot's softmax runs.
// K_j and V_j stream through a 5-stage ring; the producer walks exactly the
// same merged event order as the MMA thread, so the ring is a plain FIFO.
//
// Warp roles (384 threads, three warpgroups):
//   warps 0..3  control warpgroup, 80 registers a thread: warp 0 TMA producer,
//               warp 1 TMEM allocator + MMA issuer (warps 2, 3 idle)
//   warps 4..7  softmax + output epilogue of slot 0, 208 registers a thread
//   warps 8..11 softmax + output epilogue of slot 1 (warp w owns TMEM lanes
//               32*(w%4) .. 32*(w%4)+31)
// The launch gives 384 x 168 registers; setmaxnreg moves them from the
// control warpgroup to the softmax warpgroups (128*80 + 256*208 <= 384*168),
// which hold a whole 128-score row in registers.
// Units come from the longest-list-first order: slot s of CTA c takes units
// 2c+s, 2c+s+2G, ... (G = grid size). Every pipeline wait is bounded; on
// time-out the CTA raises its abort flag, drains, frees TMEM and records
// XATTN_ERR_TIMEOUT in the status word.
#include <cuda_bf16.h>

#include "common.cuh"
#include "ptx.cuh"

namespace xattn {
namespace {

constexpr int kThreads = 384;
constexpr int kBlk = 128;                      // B (rows per query / key block)
constexpr int kD = 128;                        // head dim
constexpr int kHalf = kBlk * 64 * 2;           // one 64-feature box: 16 KB
constexpr int kTileBytes = 2 * kHalf;          // 128 x 128 bf16: 32 KB
constexpr int kStages = 5;
constexpr int kSlots = 2;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSlotCols = 256;            // per slot: S at +0 (P aliases +0..63), O at +128
constexpr uint32_t kColO = 128;
constexpr uint32_t kIdescS = idesc_bf16_f32(kBlk, kBlk, 0, 0);
constexpr uint32_t kIdescPV = idesc_bf16_f32(kBlk, kD, 0, 1);  // V is MN-major
constexpr float kRescaleLog2 = 8.0f;           // rescale O only when the max grows by > 2^8
constexpr int kLaunchRegs = 168;               // registers a thread at launch (__launch_bounds__)
constexpr int kCtrlRegs = 80, kSoftmaxRegs = 208;
static_assert(128 * kCtrlRegs + 256 * kSoftmaxRegs <= kThreads * kLaunchRegs,
              "setmaxnreg split exceeds the registers the block is launched with");

struct Params {
  int L, NB, hq, hkv, group, causal, units;
  float scale_log2;  // log2(e) / sqrt(d)
  const int32_t* counts;
  const int32_t* idx;
  const unsigned long long* order;  // packed entries: unit | n << 32 | diag << 48
  __nv_bfloat16* O;
  float* lse;
  int* status;
  int o_store32;  // O is 32-byte aligned: rows are written with 32-byte stores
};

struct Smem {
  uint64_t kv_full[kStages], kv_empty[kStages];
  uint64_t q_full[kSlots], q_empty[kSlots];
  uint64_t s_full[kSlots], p_full[kSlots], pv_done[kSlots], o_empty[kSlots];
  uint32_t tmem_base;
  int abort;
};

// One packed work-order entry (written by the schedule kernel).
constexpr unsigned long long kEndEntry = ~0ull;

__device__ __forceinline__ unsigned long long load_entry(const Params& p, int k) {
  return k < p.units ? __ldg(p.order + k) : kEndEntry;
}
__device__ __forceinline__ int entry_unit(unsigned long long e) {
  return static_cast<int>(e & 0xFFFFFFFFull);
}
__device__ __forceinline__ int entry_count(unsigned long long e) {
  return static_cast<int>((e >> 32) & 0xFFFFull);
}
__device__ __forceinline__ bool entry_diag(unsigned long long e) { return (e >> 48) & 1ull; }

// Walks the blocks of one slot's units in order, skipping units with no block.
// The next unit's entry is always one load ahead; the producer (kList) also
// keeps the next block index of the list one load ahead.
struct Cursor {
  int k;        // position in the unit order
  int step;     // distance between this slot's units (2 * grid)
  int unit, bh, qb, n, j;
  const int32_t* list;
  int kb, kb_next;                // list[j], list[j + 1]
  unsigned long long next_entry;  // order entry at position k (before a seek)
  bool valid;
};

template <bool kList>
__device__ __forceinline__ void cursor_seek(Cursor& c, const Params& p) {
  for (;;) {
    if (c.k >= p.units) {
      c.valid = false;
      return;
    }
    const unsigned long long e = c.next_entry;
    c.next_entry = load_entry(p, c.k + c.step);  // prefetch the following unit
    const int n = entry_count(e);
    if (n > 0) {
      c.unit = entry_unit(e);
      c.bh = c.unit / p.NB;
      c.qb = c.unit % p.NB;
      c.list = p.idx + static_cast<size_t>(c.unit) * p.NB;
      c.n = n;
      c.j = 0;
      if (kList) {
        c.kb = c.list[0];
        c.kb_next = n > 1 ? c.list[1] : 0;
      }
      c.valid = true;
      return;
    }
    c.k += c.step;
  }
}

template <bool kList>
__device__ __forceinline__ void cursor_init(Cursor& c, const Params& p, int slot) {
  c.k = 2 * blockIdx.x + slot;
  c.step = 2 * gridDim.x;
  c.next_entry = load_entry(p, c.k);
  cursor_seek<kList>(c, p);
}

// Moves past the current block; returns false when the slot has no more work.
template <bool kList>
__device__ __forceinline__ bool cursor_next(Cursor& c, const Params& p) {
  if (++c.j < c.n) {
    if (kList) {
      c.kb = c.kb_next;
      if (c.j + 1 < c.n) c.kb_next = c.list[c.j + 1];
    }
    return true;
  }
  c.k += c.step;
  cursor_seek<kList>(c, p);
  return c.valid;
}

struct SlotState {
  Cursor cur;
  bool pend;       // an S was issued whose PV is still to come
  int pend_j;      // block index of that S within its unit
  uint32_t units;  // units started (first S issued)
  uint32_t blocks; // PV events done
};

struct Ring {
  int stage;
  uint32_t phase;
  long long issued;
  __device__ __forceinline__ void next() {
    if (++stage == kStages) {
      stage = 0;
      phase ^= 1;
    }
  }
};

struct Ctx {
  const Params* p;
  Smem* sm;
  uint8_t* q_smem;
  uint8_t* kv_smem;
  uint32_t tmem;
  const CUtensorMap* tmQ;
  const CUtensorMap* tmK;
  const CUtensorMap* tmV;
  volatile int* abort;
};

// S event of slot kSlot for the cursor's current block. The producer loads Q
// (first block of a unit) and K; the MMA thread issues S = Q K^T.
template <bool kMma, int kSlot>
__device__ __forceinline__ bool event_s(SlotState& st, Ring& ring, const Ctx& x) {
  const Params& p = *x.p;
  Smem* sm = x.sm;
  Cursor& c = st.cur;
  const bool first = c.j == 0;
  const bool last = c.j == c.n - 1;
  if (!kMma) {
    if (first) {
      if (!warp_wait(&sm->q_empty[kSlot], (st.units & 1) ^ 1, x.abort)) return false;
      if (elect_one()) {
        mbar_arrive_expect_tx(&sm->q_full[kSlot], kTileBytes);
        const int qrow = c.bh * p.L + c.qb * kBlk;
        tma_load_2d(x.q_smem + kSlot * kTileBytes, x.tmQ, &sm->q_full[kSlot], 0, qrow);
        tma_load_2d(x.q_smem + kSlot * kTileBytes + kHalf, x.tmQ, &sm->q_full[kSlot], 64, qrow);
      }
      __syncwarp();
    }
    if (!warp_wait(&sm->kv_empty[ring.stage], ring.phase ^ 1, x.abort)) return false;
    if (elect_one()) {
      const int kvbh = (c.bh / p.hq) * p.hkv + (c.bh % p.hq) / p.group;
      const int krow = kvbh * p.L + c.kb * kBlk;
      uint8_t* dst = x.kv_smem + ring.stage * kTileBytes;
      mbar_arrive_expect_tx(&sm->kv_full[ring.stage], kTileBytes);
      tma_load_2d(dst, x.tmK, &sm->kv_full[ring.stage], 0, krow);
      tma_load_2d(dst + kHalf, x.tmK, &sm->kv_full[ring.stage], 64, krow);
    }
    __syncwarp();
    ++ring.issued;
  } else {
    if (first && !warp_wait(&sm->q_full[kSlot], st.units & 1, x.abort)) return false;
    if (!warp_wait(&sm->kv_full[ring.stage], ring.phase, x.abort)) return false;
    tc_fence_after();
    if (elect_one()) {
      const uint32_t q_addr = smem_u32(x.q_smem + kSlot * kTileBytes);
      const uint32_t k_addr = smem_u32(x.kv_smem + ring.stage * kTileBytes);
      const uint32_t dS = x.tmem + kSlot * kSlotCols;
#pragma unroll
      for (int kk = 0; kk < kD / 16; ++kk) {
        const uint32_t off = (kk >> 2) * kHalf + (kk & 3) * 32;
        umma_ss(dS, smem_desc_sw128(q_addr + off, 16, 1024),
                smem_desc_sw128(k_addr + off, 16, 1024), kIdescS, kk > 0);
      }
      umma_commit(&sm->s_full[kSlot]);
      umma_commit(&sm->kv_empty[ring.stage]);
      if (last) umma_commit(&sm->q_empty[kSlot]);
    }
    __syncwarp();
  }
  if (first) ++st.units;
  st.pend = true;
  st.pend_j = c.j;
  ring.next();
  return true;
}

// PV event of slot kSlot's pending block (the cursor still points at it).
// The producer loads V; the MMA thread issues O += P V.
template <bool kMma, int kSlot>
__device__ __forceinline__ bool event_pv(SlotState& st, Ring& ring, const Ctx& x) {
  const Params& p = *x.p;
  Smem* sm = x.sm;
  const Cursor& c = st.cur;
  const bool first = st.pend_j == 0;
  if (!kMma) {
    if (!warp_wait(&sm->kv_empty[ring.stage], ring.phase ^ 1, x.abort)) return false;
    if (elect_one()) {
      const int kvbh = (c.bh / p.hq) * p.hkv + (c.bh % p.hq) / p.group;
      const int vrow = kvbh * p.L + c.kb * kBlk;
      uint8_t* dst = x.kv_smem + ring.stage * kTileBytes;
      mbar_arrive_expect_tx(&sm->kv_full[ring.stage], kTileBytes);
      tma_load_2d(dst, x.tmV, &sm->kv_full[ring.stage], 0, vrow);
      tma_load_2d(dst + kHalf, x.tmV, &sm->kv_full[ring.stage], 64, vrow);
    }
    __syncwarp();
    ++ring.issued;
  } else {
    if (!warp_wait(&sm->p_full[kSlot], st.blocks & 1, x.abort)) return false;
    // the unit's first PV overwrites O: the previous unit's epilogue must be done
    if (first && !warp_wait(&sm->o_empty[kSlot], ((st.units - 1) & 1) ^ 1, x.abort)) return false;
    if (!warp_wait(&sm->kv_full[ring.stage], ring.phase, x.abort)) return false;
    tc_fence_after();
    if (elect_one()) {
      const uint32_t v_addr = smem_u32(x.kv_smem + ring.stage * kTileBytes);
      const uint32_t dO = x.tmem + kSlot * kSlotCols + kColO;
      const uint32_t aP = x.tmem + kSlot * kSlotCols;
#pragma unroll
      for (int kk = 0; kk < kBlk / 16; ++kk) {
        // 16 keys per step: P columns [8kk, 8kk+8) (bf16 pairs), V rows [16kk, 16kk+16)
        umma_ts(dO, aP + kk * 8, smem_desc_sw128(v_addr + kk * 16 * 128, kHalf, 1024), kIdescPV,
                (!first || kk > 0) ? 1u : 0u);
      }
      umma_commit(&sm->pv_done[kSlot]);
      umma_commit(&sm->kv_empty[ring.stage]);
    }
    __syncwarp();
  }
  ++st.blocks;
  st.pend = false;
  ring.next();
  return true;
}

template <bool kMma>
__device__ __forceinline__ void pipeline(const Params& p, Smem* sm, uint8_t* q_smem,
                                      uint8_t* kv_smem, uint32_t tmem, const CUtensorMap* tmQ,
                                      const CUtensorMap* tmK, const CUtensorMap* tmV,
                                      volatile int* abort) {
  const Ctx x{&p, sm, q_smem, kv_smem, tmem, tmQ, tmK, tmV, abort};
  Ring ring{0, 0u, 0};
  SlotState s0{}, s1{};
  cursor_init<!kMma>(s0.cur, p, 0);
  cursor_init<!kMma>(s1.cur, p, 1);
  bool ok = true;
  if (s0.cur.valid) ok = event_s<kMma, 0>(s0, ring, x);
  if (ok && s1.cur.valid) ok = event_s<kMma, 1>(s1, ring, x);
  while (ok && (s0.pend || s1.pend)) {
    if (s0.pend) {
      ok = event_pv<kMma, 0>(s0, ring, x);
      if (ok && cursor_next<!kMma>(s0.cur, p)) ok = event_s<kMma, 0>(s0, ring, x);
    }
    if (ok && s1.pend) {
      ok = event_pv<kMma, 1>(s1, ring, x);
      if (ok && cursor_next<!kMma>(s1.cur, p)) ok = event_s<kMma, 1>(s1, ring, x);
    }
  }
  if (!ok && !kMma) {
    // wait (bounded) for the copies this thread still has in flight
    const long long nk = ring.issued < kStages ? ring.issued : kStages;
    for (long long t = 1; t <= nk; ++t) {
      const long long q = ring.issued - t;
      const uint32_t addr = smem_u32(&sm->kv_full[q % kStages]);
      const uint32_t ph = static_cast<uint32_t>((q / kStages) & 1);
      const unsigned long long t0 = globaltimer();
      while (!mbar_try_wait(addr, ph) && globaltimer() - t0 < kWaitLimitNs) {
      }
    }
    const uint32_t nu[kSlots] = {s0.units, s1.units};
    for (int s = 0; s < kSlots; ++s) {
      if (nu[s] == 0) continue;
      const uint32_t addr = smem_u32(&sm->q_full[s]);
      const unsigned long long t0 = globaltimer();
      while (!mbar_try_wait(addr, (nu[s] - 1) & 1) && globaltimer() - t0 < kWaitLimitNs) {
      }
    }
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ,
                   const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* q_smem = base;                              // kSlots tiles
  uint8_t* kv_smem = base + kSlots * kTileBytes;       // kStages tiles
  Smem* sm = reinterpret_cast<Smem*>(base + (kSlots + kStages) * kTileBytes);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm->kv_full[s], 1);
      mbar_init(&sm->kv_empty[s], 1);
    }
    for (int s = 0; s < kSlots; ++s) {
      mbar_init(&sm->q_full[s], 1);
      mbar_init(&sm->q_empty[s], 1);
      mbar_init(&sm->s_full[s], 1);
      mbar_init(&sm->p_full[s], 128);
      mbar_init(&sm->pv_done[s], 1);
      mbar_init(&sm->o_empty[s], 128);
    }
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

  if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 80;\n" ::: "memory");  // 128 x 80
    if (warp <= 1) {
      // Producer (warp 0) and MMA issuer (warp 1) walk the same merged event
      // order: S(0), S(1), { PV(0), S(0, next), PV(1), S(1, next) } ...
      // Each role runs on its whole warp; one elected lane issues the TMA
      // copies / MMAs and commits.
      if (warp == 0)
        pipeline<false>(p, sm, q_smem, kv_smem, tmem, &tmQ, &tmK, &tmV, abort);
      else
        pipeline<true>(p, sm, q_smem, kv_smem, tmem, &tmQ, &tmK, &tmV, abort);
    }
  } else {
    // ------------------------------------------------ softmax + epilogue
    asm volatile("setmaxnreg.inc.sync.aligned.u32 208;\n" ::: "memory");  // 256 x 208
    const int slot = (warp - 4) / 4;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tS = tmem + lane_addr + slot * kSlotCols;
    const uint32_t tO = tS + kColO;
    const float sl2 = p.scale_log2;
    uint32_t g = 0;  // blocks processed by this slot
    unsigned long long e_next = load_entry(p, 2 * blockIdx.x + slot);
    for (int k = 2 * blockIdx.x + slot; k < p.units; k += 2 * gridDim.x) {
      const unsigned long long e = e_next;
      e_next = load_entry(p, k + 2 * gridDim.x);  // prefetch the next unit's entry
      const int unit = entry_unit(e);
      const int bh = unit / p.NB, qb = unit % p.NB;
      const int n = entry_count(e);
      const size_t orow = static_cast<size_t>(bh) * p.L + static_cast<size_t>(qb) * kBlk + row;
      __nv_bfloat16* optr = p.O + orow * kD;
      if (n <= 0) {
        const uint4 z = make_uint4(0, 0, 0, 0);
        for (int c = 0; c < kD / 8; ++c) reinterpret_cast<uint4*>(optr)[c] = z;
        if (p.lse) p.lse[orow] = -INFINITY;
        continue;
      }
      // a causal list is ascending and ends at most at qb: only its last
      // block can be the diagonal one (flagged in the order entry)
      const bool last_is_diag = entry_diag(e);
      float m_run = -INFINITY;  // running max of scaled logits (log2 units)
      float l_run = 0.f;
      bool failed = false;
      for (int j = 0; j < n; ++j, ++g) {
        const bool diag = last_is_diag && j == n - 1;
        if (!warp_wait(&sm->s_full[slot], g & 1, abort)) {
          failed = true;
          break;
        }
        tc_fence_after();
        uint32_t sv[4][32];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(tS + c * 32, sv[c]);
        tmem_ld_wait();
        float mx = -INFINITY;
        if (diag) {
#pragma unroll
          for (int c = 0; c < 4; ++c)
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (c * 32 + i > row) sv[c][i] = __float_as_uint(-INFINITY);
        }
        {
          // 8 independent partial maxima over 16 scores each (three-input
          // max: 8 instructions a group), then a short tree
          float pm[8];
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const uint32_t* g16 = &sv[q >> 1][(q & 1) * 16];
            float m = fmax3(__uint_as_float(g16[0]), __uint_as_float(g16[1]),
                            __uint_as_float(g16[2]));
#pragma unroll
            for (int i = 3; i < 15; i += 2)
              m = fmax3(m, __uint_as_float(g16[i]), __uint_as_float(g16[i + 1]));
            pm[q] = fmaxf(m, __uint_as_float(g16[15]));
          }
          mx = fmax3(fmax3(pm[0], pm[1], pm[2]), fmax3(pm[3], pm[4], pm[5]),
                     fmaxf(pm[6], pm[7]));
        }
        const float m_new = fmaxf(m_run, mx * sl2);
        const bool need = m_new > m_run + kRescaleLog2;
        const bool any_need = __any_sync(0xffffffffu, need);
        const float alpha = need ? ex2(m_run - m_new) : 1.0f;
        if (need) {
          l_run *= alpha;
          m_run = m_new;
        }
        const unsigned long long scale2 = f2_pack(sl2, sl2);
        const unsigned long long negm2 = f2_pack(-m_run, -m_run);
        unsigned long long lsum2[4];   // 4 independent pair-accumulators
#pragma unroll
        for (int q = 0; q < 4; ++q) lsum2[q] = f2_pack(0.f, 0.f);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          // keys [64h, 64h + 64) -> bf16 pairs in TMEM columns [32h, 32h + 32)
          uint32_t pk[32];
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const int e = 64 * h + 2 * c;
            const unsigned long long x2 =
                f2_pack(__uint_as_float(sv[e >> 5][e & 31]),
                        __uint_as_float(sv[(e + 1) >> 5][(e + 1) & 31]));
            float a0, a1;
            f2_unpack(f2_fma(x2, scale2, negm2), a0, a1);
            const float p0 = ex2(a0);
            const float p1 = ex2(a1);
            lsum2[c & 3] = f2_add(lsum2[c & 3], f2_pack(p0, p1));
            pk[c] = pack_bf16x2(p0, p1);
          }
          tmem_st32(tS + 32 * h, pk);
        }
        float ls0, ls1, ls2, ls3, ls4, ls5, ls6, ls7;
        f2_unpack(lsum2[0], ls0, ls1);
        f2_unpack(lsum2[1], ls2, ls3);
        f2_unpack(lsum2[2], ls4, ls5);
        f2_unpack(lsum2[3], ls6, ls7);
        l_run += ((ls0 + ls1) + (ls2 + ls3)) + ((ls4 + ls5) + (ls6 + ls7));
        if (any_need && j > 0) {
          // O holds PV_0..PV_{j-1}: wait for the last one, then rescale in place
          // (PV_j cannot start before this thread arrives on p_full below)
          if (!warp_wait(&sm->pv_done[slot], (g - 1) & 1, abort)) {
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
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&sm->p_full[slot]);
      }
      if (failed) break;
      // ---- epilogue: O / l -> bf16 rows
      if (!warp_wait(&sm->pv_done[slot], (g - 1) & 1, abort)) break;
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
        if (p.o_store32) {
          // full 32-byte sectors, half the store instructions
          st_global_v8(optr + c * 32, w);
          st_global_v8(optr + c * 32 + 16, w + 8);
        } else {
          uint4* dst = reinterpret_cast<uint4*>(optr + c * 32);
#pragma unroll
          for (int i = 0; i < 4; ++i)
            dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
        }
      }
      if (p.lse) p.lse[orow] = (m_run + lg2(l_run)) * 0.69314718055994531f;
      tc_fence_before();
      mbar_arrive(&sm->o_empty[slot]);
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
                           const unsigned long long* order, void* O, float* lse, int* status,
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
  p.o_store32 = (reinterpret_cast<uintptr_t>(O) & 31u) == 0;
  const size_t smem = 1024 + kTileBytes * (kSlots + kStages) + sizeof(Smem);
  cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  int grid = num_sms;
  const int need = (p.units + 1) / 2;
  if (grid > need) grid = need;
  if (grid < 1) grid = 1;
  attn_tc_kernel<<<grid, kThreads, smem, st>>>(tmQ, tmK, tmV, p);
  return cudaGetLastError();
}

}  // namespace xattn
