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
// One persistent CTA per SM takes units one at a time, in longest-list-first
// order. TMEM holds two S buffers (block parity) and two O buffers (unit
// parity). The MMA thread keeps two S ahead of the softmax -- per CTA its
// order is S(0), S(1), then {PV(t), S(t+2)} over the CTA's blocks t, across
// units -- so the softmax warpgroup runs block after block without waiting
// for the tensor core. The producer walks the same order, so the 5-stage K/V
// ring is a plain FIFO; Q tiles are double-buffered by unit parity.
//
// A unit's output is written by a separate epilogue warpgroup: at the unit's
// end the softmax warpgroup leaves each row's running max and sum in shared
// memory and goes on with the next unit; the epilogue warpgroup waits for the
// unit's last PV, then normalises and stores O and frees the O buffer.
//
// Warp roles (384 threads, three warpgroups):
//   warps 0..3  control warpgroup, 80 registers a thread: warp 0 TMA producer,
//               warp 1 TMEM allocator + MMA issuer (warps 2, 3 idle). Both
//               issuing roles run on their whole warp; one elected lane issues.
//   warps 4..7  softmax, 208 registers a thread (a whole 128-score row)
//   warps 8..11 output epilogue, 80 registers a thread
//   (warp w owns TMEM lanes 32*(w%4) .. 32*(w%4)+31)
// The launch gives 384 x 168 registers; setmaxnreg redistributes them
// (128*80 + 128*208 + 128*80 <= 384*168). Every wait is bounded; on time-out
// the CTA raises its abort flag, drains, frees TMEM and records
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
constexpr int kStages = 5;                     // K/V ring
constexpr int kQBufs = 2;                      // Q tiles (unit parity)
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 256;                // S buffers at 0, 128; O buffers at 256, 384
constexpr uint32_t kIdescS = idesc_bf16_f32(kBlk, kBlk, 0, 0);
constexpr uint32_t kIdescPV = idesc_bf16_f32(kBlk, kD, 0, 1);  // V is MN-major
constexpr float kRescaleLog2 = 8.0f;           // rescale O only when the max grows by > 2^8
constexpr int kLaunchRegs = 168;               // registers a thread at launch (__launch_bounds__)
constexpr int kCtrlRegs = 80, kSoftmaxRegs = 208, kEpiRegs = 80;
static_assert(128 * (kCtrlRegs + kSoftmaxRegs + kEpiRegs) <= kThreads * kLaunchRegs,
              "setmaxnreg split exceeds the registers the block is launched with");

struct Params {
  int L, NB, hq, hkv, group, causal, units;
  int tail;          // tokens of the last block (B unless the length is ragged)
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
  uint64_t q_full[kQBufs], q_empty[kQBufs];
  uint64_t s_full[2], p_full[2], pv_done[2];  // by block parity
  uint64_t o_full[2], o_empty[2];             // by unit parity: last PV done / O read out
  uint64_t ml_full[2];                        // by unit parity: row max / sum written
  float ml[2][2][kBlk];                       // [unit parity][max, sum][row]
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
// The unit's last listed block needs a column mask: the diagonal block
// (causal: keys after the query), or the short last block (non-causal: keys
// at or past L).
__device__ __forceinline__ bool entry_masked(unsigned long long e) { return (e >> 48) & 1ull; }

// Walks the blocks of this CTA's units in order, skipping units with no block.
// The next unit's entry is always one load ahead; the producer (kList) also
// keeps the next block index of the list one load ahead.
struct Cursor {
  int k;        // position in the unit order
  int step;     // distance between this CTA's units (the grid size)
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
__device__ __forceinline__ void cursor_init(Cursor& c, const Params& p) {
  c.k = blockIdx.x;
  c.step = gridDim.x;
  c.next_entry = load_entry(p, c.k);
  cursor_seek<kList>(c, p);
}

// Moves past the current block; returns false when the CTA has no more work.
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

// A block whose S has been issued and whose PV has not (at most two). Named,
// not indexed, so it stays in registers.
struct BlockInfo {
  int kvrow;    // first K/V row of the key block in the [bh*L, d] view (producer)
  uint32_t u;   // unit sequence number within the CTA (Q / O buffer parity)
  bool first;   // first block of its unit
  bool last;    // last block of its unit
};

struct Fifo {
  BlockInfo b0, b1;
  int n;
  __device__ __forceinline__ void push(const BlockInfo& b) {
    if (n == 0)
      b0 = b;
    else
      b1 = b;
    ++n;
  }
  __device__ __forceinline__ void pop() {
    b0 = b1;
    --n;
  }
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

struct PipeState {
  Cursor cur;       // next block whose S is to be issued
  Fifo fifo;        // blocks with S issued and PV not yet issued
  uint32_t ts;      // blocks with S issued (S buffer = ts & 1)
  uint32_t tpv;     // blocks with PV issued
  uint32_t units;   // units started on the S side
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

// S event for the block at the cursor. The producer loads Q (first block of a
// unit) and K; the MMA thread issues S_t = Q K^T into S buffer t & 1.
template <bool kMma>
__device__ __forceinline__ bool event_s(PipeState& st, Ring& ring, const Ctx& x) {
  const Params& p = *x.p;
  Smem* sm = x.sm;
  const Cursor& c = st.cur;
  BlockInfo b;
  b.first = c.j == 0;
  b.last = c.j == c.n - 1;
  if (b.first) ++st.units;
  b.u = st.units - 1;
  b.kvrow = 0;
  const uint32_t qb = b.u & 1;  // Q buffer
  if (!kMma) {
    const int kvbh = (c.bh / p.hq) * p.hkv + (c.bh % p.hq) / p.group;
    b.kvrow = kvbh * p.L + c.kb * kBlk;
    if (b.first) {
      if (!warp_wait(&sm->q_empty[qb], ((b.u >> 1) & 1) ^ 1, x.abort)) return false;
      if (elect_one()) {
        const int qrow = c.bh * p.L + c.qb * kBlk;
        mbar_arrive_expect_tx(&sm->q_full[qb], kTileBytes);
        tma_load_2d(x.q_smem + qb * kTileBytes, x.tmQ, &sm->q_full[qb], 0, qrow);
        tma_load_2d(x.q_smem + qb * kTileBytes + kHalf, x.tmQ, &sm->q_full[qb], 64, qrow);
      }
      __syncwarp();
    }
    if (!warp_wait(&sm->kv_empty[ring.stage], ring.phase ^ 1, x.abort)) return false;
    if (elect_one()) {
      uint8_t* dst = x.kv_smem + ring.stage * kTileBytes;
      mbar_arrive_expect_tx(&sm->kv_full[ring.stage], kTileBytes);
      tma_load_2d(dst, x.tmK, &sm->kv_full[ring.stage], 0, b.kvrow);
      tma_load_2d(dst + kHalf, x.tmK, &sm->kv_full[ring.stage], 64, b.kvrow);
    }
    __syncwarp();
    ++ring.issued;
  } else {
    if (b.first && !warp_wait(&sm->q_full[qb], (b.u >> 1) & 1, x.abort)) return false;
    if (!warp_wait(&sm->kv_full[ring.stage], ring.phase, x.abort)) return false;
    tc_fence_after();
    const uint32_t sb = st.ts & 1;  // S buffer
    if (elect_one()) {
      const uint32_t q_addr = smem_u32(x.q_smem + qb * kTileBytes);
      const uint32_t k_addr = smem_u32(x.kv_smem + ring.stage * kTileBytes);
      const uint32_t dS = x.tmem + sb * kBlk;
#pragma unroll
      for (int kk = 0; kk < kD / 16; ++kk) {
        const uint32_t off = (kk >> 2) * kHalf + (kk & 3) * 32;
        umma_ss(dS, smem_desc_sw128(q_addr + off, 16, 1024),
                smem_desc_sw128(k_addr + off, 16, 1024), kIdescS, kk > 0);
      }
      umma_commit(&sm->s_full[sb]);
      umma_commit(&sm->kv_empty[ring.stage]);
      if (b.last) umma_commit(&sm->q_empty[qb]);
    }
    __syncwarp();
  }
  st.fifo.push(b);
  ++st.ts;
  ring.next();
  return true;
}

// PV event for the oldest block in flight. The producer loads V; the MMA
// thread issues O_u += P_t V_t (O buffer = unit parity).
template <bool kMma>
__device__ __forceinline__ bool event_pv(PipeState& st, Ring& ring, const Ctx& x) {
  Smem* sm = x.sm;
  const BlockInfo b = st.fifo.b0;
  const uint32_t sb = st.tpv & 1;  // S / P buffer of this block
  const uint32_t ob = b.u & 1;     // O buffer of its unit
  if (!kMma) {
    if (!warp_wait(&sm->kv_empty[ring.stage], ring.phase ^ 1, x.abort)) return false;
    if (elect_one()) {
      uint8_t* dst = x.kv_smem + ring.stage * kTileBytes;
      mbar_arrive_expect_tx(&sm->kv_full[ring.stage], kTileBytes);
      tma_load_2d(dst, x.tmV, &sm->kv_full[ring.stage], 0, b.kvrow);
      tma_load_2d(dst + kHalf, x.tmV, &sm->kv_full[ring.stage], 64, b.kvrow);
    }
    __syncwarp();
    ++ring.issued;
  } else {
    if (!warp_wait(&sm->p_full[sb], (st.tpv >> 1) & 1, x.abort)) return false;
    // the unit's first PV overwrites its O buffer: the epilogue of the unit
    // that used it before (two units back) must have read it out
    if (b.first && !warp_wait(&sm->o_empty[ob], ((b.u >> 1) & 1) ^ 1, x.abort)) return false;
    if (!warp_wait(&sm->kv_full[ring.stage], ring.phase, x.abort)) return false;
    tc_fence_after();
    if (elect_one()) {
      const uint32_t v_addr = smem_u32(x.kv_smem + ring.stage * kTileBytes);
      const uint32_t dO = x.tmem + kColO + ob * kD;
      const uint32_t aP = x.tmem + sb * kBlk;
#pragma unroll
      for (int kk = 0; kk < kBlk / 16; ++kk) {
        // 16 keys per step: P columns [8kk, 8kk+8) (bf16 pairs), V rows [16kk, 16kk+16)
        umma_ts(dO, aP + kk * 8, smem_desc_sw128(v_addr + kk * 16 * 128, kHalf, 1024), kIdescPV,
                (!b.first || kk > 0) ? 1u : 0u);
      }
      umma_commit(&sm->pv_done[sb]);
      umma_commit(&sm->kv_empty[ring.stage]);
      if (b.last) umma_commit(&sm->o_full[ob]);
    }
    __syncwarp();
  }
  st.fifo.pop();
  ++st.tpv;
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
  PipeState st{};
  cursor_init<!kMma>(st.cur, p);
  bool ok = true;
  // two S ahead of the first PV
  for (int a = 0; a < 2 && ok && st.cur.valid; ++a) {
    ok = event_s<kMma>(st, ring, x);
    if (ok) cursor_next<!kMma>(st.cur, p);
  }
  while (ok && st.fifo.n > 0) {
    ok = event_pv<kMma>(st, ring, x);
    if (ok && st.cur.valid) {
      ok = event_s<kMma>(st, ring, x);
      if (ok) cursor_next<!kMma>(st.cur, p);
    }
  }
  if (!ok && !kMma) {
    // wait (bounded) for the copies this warp still has in flight
    const long long nk = ring.issued < kStages ? ring.issued : kStages;
    for (long long t = 1; t <= nk; ++t) {
      const long long q = ring.issued - t;
      const uint32_t addr = smem_u32(&sm->kv_full[q % kStages]);
      const uint32_t ph = static_cast<uint32_t>((q / kStages) & 1);
      const unsigned long long t0 = globaltimer();
      while (!mbar_try_wait(addr, ph) && globaltimer() - t0 < kWaitLimitNs) {
      }
    }
    for (uint32_t u = st.units > 2 ? st.units - 2 : 0; u < st.units; ++u) {
      const uint32_t addr = smem_u32(&sm->q_full[u & 1]);
      const unsigned long long t0 = globaltimer();
      while (!mbar_try_wait(addr, (u >> 1) & 1) && globaltimer() - t0 < kWaitLimitNs) {
      }
    }
  }
}

// Softmax warpgroup: P for every block, running max / sum per row.
__device__ __forceinline__ void softmax_role(const Params& p, Smem* sm, uint32_t tmem, int warp,
                                             int lane, volatile int* abort) {
  const int quarter = warp & 3;
  const int row = quarter * 32 + lane;
  const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
  const float sl2 = p.scale_log2;
  uint32_t g = 0;  // blocks processed by this CTA
  uint32_t u = 0;  // non-empty units processed
  unsigned long long e_next = load_entry(p, blockIdx.x);
  for (int k = blockIdx.x; k < p.units; k += gridDim.x) {
    const unsigned long long e = e_next;
    e_next = load_entry(p, k + gridDim.x);  // prefetch the next unit's entry
    const int n = entry_count(e);
    if (n <= 0) continue;                   // the epilogue warpgroup writes it
    const uint32_t ob = u & 1;
    const uint32_t tO = tmem + lane_addr + kColO + ob * kD;
    // lists are ascending: only the last block can be the diagonal one
    // (causal, ends at most at qb) or the short last one (flagged in the
    // order entry). Keep columns <= lim of that block.
    const bool last_masked = entry_masked(e);
    const int lim = p.causal ? row : p.tail - 1;
    float m_run = -INFINITY;  // running max of scaled logits (log2 units)
    float l_run = 0.f;
    for (int j = 0; j < n; ++j, ++g) {
      const bool masked = last_masked && j == n - 1;
      const uint32_t sb = g & 1;
      const uint32_t tS = tmem + lane_addr + sb * kBlk;
      if (!warp_wait(&sm->s_full[sb], (g >> 1) & 1, abort)) return;
      tc_fence_after();
      uint32_t sv[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(tS + c * 32, sv[c]);
      tmem_ld_wait();
      if (masked) {
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (c * 32 + i > lim) sv[c][i] = __float_as_uint(-INFINITY);
      }
      float mx;
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
          const int e0 = 64 * h + 2 * c;
          const unsigned long long x2 =
              f2_pack(__uint_as_float(sv[e0 >> 5][e0 & 31]),
                      __uint_as_float(sv[(e0 + 1) >> 5][(e0 + 1) & 31]));
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
        if (!warp_wait(&sm->pv_done[(g - 1) & 1], ((g - 1) >> 1) & 1, abort)) return;
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
      mbar_arrive(&sm->p_full[sb]);
    }
    // hand the row's max and sum to the epilogue warpgroup; the slot was last
    // used two units back, whose epilogue must have read it (o_empty)
    if (!warp_wait(&sm->o_empty[ob], ((u >> 1) & 1) ^ 1, abort)) return;
    sm->ml[ob][0][row] = m_run;
    sm->ml[ob][1][row] = l_run;
    mbar_arrive(&sm->ml_full[ob]);
    ++u;
  }
}

// Epilogue warpgroup: O / l -> bf16 rows (and lse) for every unit.
__device__ __forceinline__ void epilogue_role(const Params& p, Smem* sm, uint32_t tmem, int warp,
                                              int lane, volatile int* abort) {
  const int quarter = warp & 3;
  const int row = quarter * 32 + lane;
  const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
  uint32_t u = 0;
  unsigned long long e_next = load_entry(p, blockIdx.x);
  for (int k = blockIdx.x; k < p.units; k += gridDim.x) {
    const unsigned long long e = e_next;
    e_next = load_entry(p, k + gridDim.x);
    const int unit = entry_unit(e);
    const int bh = unit / p.NB, qb = unit % p.NB;
    const int n = entry_count(e);
    const size_t orow = static_cast<size_t>(bh) * p.L + static_cast<size_t>(qb) * kBlk + row;
    __nv_bfloat16* optr = p.O + orow * kD;
    // rows past L in a short last block belong to no query: nothing is stored
    const bool row_valid = qb < p.NB - 1 || row < p.tail;
    if (n <= 0) {
      if (!row_valid) continue;
      const uint4 z = make_uint4(0, 0, 0, 0);
      for (int c = 0; c < kD / 8; ++c) reinterpret_cast<uint4*>(optr)[c] = z;
      if (p.lse) p.lse[orow] = -INFINITY;
      continue;
    }
    const uint32_t ob = u & 1;
    const uint32_t par = (u >> 1) & 1;
    if (!warp_wait(&sm->ml_full[ob], par, abort)) return;
    const float m_run = sm->ml[ob][0][row];
    const float l_run = sm->ml[ob][1][row];
    if (!warp_wait(&sm->o_full[ob], par, abort)) return;
    tc_fence_after();
    const uint32_t tO = tmem + lane_addr + kColO + ob * kD;
    const float inv = l_run > 0.f ? 1.0f / l_run : 0.f;
#pragma unroll 1
    for (int c = 0; c < kD / 32; ++c) {
      uint32_t v[32];
      tmem_ld32(tO + c * 32, v);  // warp-collective: every lane loads
      tmem_ld_wait();
      if (!row_valid) continue;
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
    if (p.lse && row_valid) p.lse[orow] = (m_run + lg2(l_run)) * 0.69314718055994531f;
    tc_fence_before();
    mbar_arrive(&sm->o_empty[ob]);
    ++u;
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ,
                   const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const Params p) {
  // The 128-byte swizzled tiles need 1024-byte alignment. The dynamic shared
  // memory of a kernel without static shared variables starts aligned; the
  // check below reports a misaligned base instead of relying on it, since
  // the tiles use nearly all of the 227 KB.
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if ((smem_u32(smem_raw) & 1023u) != 0) {
    if (threadIdx.x == 0) atomicExch(p.status, kStatusTimeout);
    return;
  }
  uint8_t* base = smem_raw;
  uint8_t* q_smem = base;                              // kQBufs tiles
  uint8_t* kv_smem = base + kQBufs * kTileBytes;       // kStages tiles
  Smem* sm = reinterpret_cast<Smem*>(base + (kQBufs + kStages) * kTileBytes);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm->kv_full[s], 1);
      mbar_init(&sm->kv_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sm->q_full[s], 1);
      mbar_init(&sm->q_empty[s], 1);
      mbar_init(&sm->s_full[s], 1);
      mbar_init(&sm->p_full[s], 128);
      mbar_init(&sm->pv_done[s], 1);
      mbar_init(&sm->o_full[s], 1);
      mbar_init(&sm->o_empty[s], 128);
      mbar_init(&sm->ml_full[s], 128);
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
    if (warp == 0)
      pipeline<false>(p, sm, q_smem, kv_smem, tmem, &tmQ, &tmK, &tmV, abort);
    else if (warp == 1)
      pipeline<true>(p, sm, q_smem, kv_smem, tmem, &tmQ, &tmK, &tmV, abort);
  } else if (warp < 8) {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 208;\n" ::: "memory");  // 128 x 208
    softmax_role(p, sm, tmem, warp, lane, abort);
  } else {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 80;\n" ::: "memory");  // 128 x 80
    epilogue_role(p, sm, tmem, warp, lane, abort);
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
  p.tail = D.tail;
  p.scale_log2 = static_cast<float>(1.4426950408889634 / sqrt(double(D.d)));
  p.counts = counts;
  p.idx = idx;
  p.order = order;
  p.O = static_cast<__nv_bfloat16*>(O);
  p.lse = lse;
  p.status = status;
  p.o_store32 = (reinterpret_cast<uintptr_t>(O) & 31u) == 0;
  const size_t smem = kTileBytes * (kQBufs + kStages) + sizeof(Smem);
  cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  int grid = num_sms;
  if (grid > p.units) grid = p.units;
  if (grid < 1) grid = 1;
  attn_tc_kernel<<<grid, kThreads, smem, st>>>(tmQ, tmK, tmV, p);
  return cudaGetLastError();
}

}  // namespace xattn
