// Forward of the QLoRA linear for a few tokens (M <= 16), for one linear or a
// group of linears in one launch:
//   Y_p = X_p W'_p^T + sU_p B_p^T,   sU_p = bf16_rn(s_p X_p A_p^T)
// ("QLoRA, in depth", section "The mechanism in brief": y = W x + (alpha/r)
// B A x with W dequantised for the matmul; "QLoRA and Fine-Tuning on One
// Consumer GPU", section "The idea in one line": each weight tile is
// dequantised only for the moment it is used).
//
// With a handful of tokens the product does 2 M flops per weight, so the
// launch is bound by streaming the packed weight (0.516 B per weight) and by
// the work of turning codes into bf16 operands, not by the tensor cores. The
// design keeps that work off the ALU pipe and HBM busy:
//
// * A producer warp streams each chunk of 8 NF4 blocks x 128 weight rows
//   (32 KB of codes) into a shared-memory ring with two 2-D TMA copies
//   (128-byte swizzle) and the chunk's activations with two more (token rows
//   beyond M arrive as zeros), so HBM sees whole 128-byte row segments and no
//   warp holds loads in flight in its registers. The chunk's 8-bit block
//   constants and second-level constants arrive in the same ring (cp.async,
//   completing on the chunk's barrier); the consumer warps form the block
//   scales of their own rows from there.
// * Every code byte becomes a bf16 pair with one PRMT and one shared-memory
//   load: a 256-entry table of (level[hi nibble], level[lo nibble]) pairs,
//   one copy per lane in that lane's own bank (64 KB, each entry's row of 256
//   bytes half used), so the 32 lookups of a warp never conflict.
// * The table holds unscaled levels, so the block constant is applied to
//   the fp32 partial sum of each 64-weight block (one FFMA per accumulator
//   element per block) instead of to each weight. The operands the tensor
//   cores see are bf16(lambda * level) and the block scale is
//   fp32(q8 * d) / lambda; lambda = 1.43675 is the power-free factor that
//   minimises the relative bf16 rounding error of the 14 levels other than
//   0 and +-1 (rms 1.4e-3 -> 0.85e-3). The product therefore equals
//   X W'^T up to bf16 rounding of the levels rather than of level * scale.
// * Each 64-weight block feeds the warp-level MMA (m16n8k16, fp32
//   accumulate) as four k-steps; inside a block the K order is permuted so
//   that a lane's 8 code bytes of a row are exactly its A-fragment pairs, and
//   its activation fragment is 32 contiguous bytes of one token row in
//   shared memory (padded rows: conflict-free 16-byte loads). MMA rows g and
//   g + 8 of a 16-row tile are weight rows 2g and 2g + 1, so that under the
//   128-byte swizzle the 8-byte code reads of a warp fall in distinct banks.
// * Work is split evenly over one persistent CTA per SM as a list of
//   (linear, 128-row tile, 64-K block) units, stream-K style. A tile cut
//   between CTAs is finished by the CTA holding its first block (for that
//   CTA the tile is its last segment); every later contributor has the tile
//   as its first segment and publishes its fp32 partial early in its range,
//   flagged with a value unique to the launch. Partials are added in CTA
//   order, so results do not depend on timing.
// * Epilogue warps take each finished segment's sums from shared memory,
//   publish or finish the tile while the consumers stream on, and add the
//   LoRA term sU B^T in fp32 before the single bf16 rounding of Y.
// * sU = bf16(s X A^T) is formed in the same launch: at the start the
//   epilogue warps of all CTAs split X A^T into 256-K pieces, the last piece
//   of a linear to arrive sums them in order and publishes sU, and tiles wait
//   (bounded) for it before their LoRA term.
//
// Every wait is bounded (about one second): a wait that runs out sets
// QLORA_ERR_TIMEOUT in the status word and the CTA leaves. The two counters
// per linear (pieces of X A^T done, tiles that have used them) are plain
// atomic adds on a zero-initialised page, reset to zero by their last user;
// the published-partial flags carry a value unique to the launch and are
// cleared by the CTA that reads them. A launch thus leaves the workspace as it
// found it, and a captured launch can be replayed.
#include <atomic>
#include <chrono>

#include "qlora_device.cuh"

namespace qlora {

bool encode_2d(CUtensorMap *map, CUtensorMapDataType dtype, const void *base, uint64_t inner, uint64_t outer,
               uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swizzle);

namespace {

constexpr int kSmMaxProblems = 8;
constexpr int kSmTileRows = 128;
constexpr int kConsumerWarps = 8;                    // 4 row groups x 2 K slices
constexpr int kProducerWarp = 8;
constexpr int kEpiWarp0 = 9;
constexpr int kEpiWarps = 4;
constexpr int kSmThreads = (kEpiWarp0 + kEpiWarps) * 32;   // 416
constexpr int kChunkBlocks = 8;                      // NF4 blocks (of 64 weights) per chunk
constexpr uint32_t kCodeSlot = kSmTileRows * kChunkBlocks * 32;   // 32 KB of codes per chunk
constexpr int kUnitK = 128;                          // K per piece of X A^T (two NF4 blocks)
constexpr uint32_t kLutBytes = 65536;                // 256 entries x 256 B (32 lanes x 4 B + unused half)
constexpr int kMaxSlots = 3;
constexpr float kLambda = 1.43675f;
constexpr float kInvLambda = 1.0f / 1.43675f;
constexpr uint32_t kEpiBar = 1;                      // named barrier of the epilogue warps

__constant__ float c_levels[16] = QLORA_NF4_LEVELS;

struct SmProblem {
  const uint8_t *codes;
  const uint8_t *scale8;
  const float *scale2;
  const uint16_t *X;       // [M, K]
  const uint16_t *A;       // [r, K], or null when sU_in is given
  const uint16_t *B;       // [N, r]
  const uint16_t *sU_in;   // [M, r] or null
  uint16_t *Y;             // [M, N]
  uint16_t *sU;            // [M, r], written when A is given
  float *upart;            // [uchunks][16 * r16][MP] partials of X A^T
  int64_t w_unit0;         // first unit of this linear in the launch's list
  int32_t N, K, kblocks, tiles, r, uchunks, u_unit0;
  float s;
};

struct SmParams {
  CUtensorMap tm_codes[kSmMaxProblems];   // codes of each linear as u8 [N][K/2], 128 x 128-byte boxes, swizzled
  CUtensorMap tm_x[kSmMaxProblems];       // activations as bf16 [M][K], boxes of MP tokens x 256
  SmProblem p[kSmMaxProblems];
  int32_t count, M;
  int64_t w_units;
  int32_t u_units;
  uint64_t epoch;          // launch value, 1 <= epoch < 2^44
  uint64_t *flags;         // [grid]: a contributor's partial is published
  float *slots;            // [grid][MP][128]: published partials
  unsigned long long *ucnt;    // [count]: pieces of X A^T done (zero at launch)
  unsigned long long *ucons;   // [count]: tiles that have used them (zero at launch)
  int32_t *status;
  int32_t pdl;
};

// ---- small PTX helpers ------------------------------------------------------
// Asynchronous copies global -> shared of 8 bytes, and of 4 bytes of which
// the first `src_bytes` are read (the rest zero-filled; 0 reads nothing).
__device__ __forceinline__ void cp_async_8(uint32_t saddr, const void *g) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(saddr), "l"(g) : "memory");
}
__device__ __forceinline__ void cp_async_4(uint32_t saddr, const void *g, uint32_t src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(saddr), "l"(g), "r"(src_bytes) : "memory");
}
// One arrival on `bar` once this thread's earlier cp.async copies are done.
__device__ __forceinline__ void cp_async_arrive(uint64_t *bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ uint32_t lds_u32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}
__device__ __forceinline__ uint4 lds_u128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}
// D = A B (C = 0) and D += A B for m16n8k16 bf16 -> fp32.
__device__ __forceinline__ void mma_zero(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%10,%10,%10,%10};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(0.f));
}
__device__ __forceinline__ void mma_acc(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                        uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ uint32_t dyn_smem_size() {
  uint32_t v;
  asm("mov.u32 %0, %%dynamic_smem_size;" : "=r"(v));
  return v;
}

// Bounded mbarrier waits of this kernel. The waits are short and frequent
// (one per chunk), so they poll with try_wait instead of asking the hardware
// to suspend the thread: a thread suspended with a long time hint was seen to
// resume tens of microseconds after its phase had completed. `backoff_ns`
// lets roles that wait long (the epilogue) yield issue slots between polls.
// After kWaitLimitNs without progress the CTA's abort flag and the TIMEOUT
// status are raised and false is returned.
__device__ __forceinline__ bool bar_wait(uint64_t *bar, uint32_t parity, volatile int *abort_flag, int32_t *status,
                                         uint32_t backoff_ns = 0) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t n = 1;; ++n) {
    if (backoff_ns) __nanosleep(backoff_ns);
    if (mbar_try_wait(bar, parity)) return true;
    if ((n & 255) == 0) {
      if (*abort_flag) return false;
      if (global_timer_ns() - t0 > kWaitLimitNs) {
        *abort_flag = 1;
        set_status(status, 6 /* QLORA_ERR_TIMEOUT */);
        return false;
      }
    }
  }
}

// Bounded wait until *w == v (GPU scope acquire); false on timeout.
__device__ __forceinline__ bool wait_word(const uint64_t *w, uint64_t v, volatile int *abort_flag, int32_t *status) {
  if (ld_acquire_gpu_u64(w) == v) return true;
  const uint64_t t0 = global_timer_ns();
  for (;;) {
    __nanosleep(64);
    if (ld_acquire_gpu_u64(w) == v) return true;
    if (*abort_flag) return false;
    if (global_timer_ns() - t0 > kWaitLimitNs) {
      *abort_flag = 1;
      set_status(status, 6 /* QLORA_ERR_TIMEOUT */);
      return false;
    }
  }
}

// ---- the unit list ----------------------------------------------------------
__device__ __forceinline__ int problem_of(const SmParams &P, int64_t u) {
  int p = 0;
#pragma unroll 1
  for (int i = 1; i < P.count; ++i)
    if (u >= P.p[i].w_unit0) p = i;
  return p;
}

// CTA whose range [b U / G, (b + 1) U / G) holds unit u.
__device__ __forceinline__ int cta_of(int64_t u, int64_t U, int64_t G) {
  return static_cast<int>(((u + 1) * G - 1) / U);
}

struct Chunk {
  int p, tile;
  int seg_lo, seg_hi;     // the segment: blocks [seg_lo, seg_hi) of the tile
  int kbA;                // chunk start aligned down to the chunk size
  int kb_s, kb_e;         // blocks of this chunk
  bool last;              // last chunk of its segment
};

struct Walk {
  int64_t u, ue;
  int p, tile, kb_lo, kb_hi, kb;
};

__device__ __forceinline__ void walk_init(Walk &w, int64_t ub, int64_t ue) {
  w.u = ub;
  w.ue = ue;
  w.p = w.tile = w.kb_lo = w.kb_hi = w.kb = 0;
}

template <int C>
__device__ __forceinline__ bool walk_next(const SmParams &P, Walk &w, Chunk &c) {
  if (w.kb >= w.kb_hi) {
    if (w.u >= w.ue) return false;
    const int p = problem_of(P, w.u);
    const SmProblem &q = P.p[p];
    const int64_t local = w.u - q.w_unit0;
    const int tile = static_cast<int>(local / q.kblocks);
    const int kb_lo = static_cast<int>(local - static_cast<int64_t>(tile) * q.kblocks);
    const int64_t tile_end = q.w_unit0 + static_cast<int64_t>(tile + 1) * q.kblocks;
    const int64_t seg_end = w.ue < tile_end ? w.ue : tile_end;
    w.p = p;
    w.tile = tile;
    w.kb_lo = kb_lo;
    w.kb_hi = kb_lo + static_cast<int>(seg_end - w.u);
    w.kb = kb_lo;
    w.u = seg_end;
  }
  c.p = w.p;
  c.tile = w.tile;
  c.seg_lo = w.kb_lo;
  c.seg_hi = w.kb_hi;
  c.kbA = (w.kb / C) * C;
  c.kb_s = w.kb;
  c.kb_e = c.kbA + C < w.kb_hi ? c.kbA + C : w.kb_hi;
  c.last = c.kb_e == w.kb_hi;
  w.kb = c.kb_e;
  return true;
}

// ---- shared-memory layout -----------------------------------------------------
// [level table 64 KB][codes ring][activation ring][constants ring][epilogue
// buffers][sU][partial sums][barriers], from the start of dynamic shared memory.
template <int MP>
struct Layout {
  static constexpr int C = kChunkBlocks;
  static constexpr int NS = MP == 8 ? 3 : 2;                // ring depth
  static constexpr uint32_t XBOX = MP * 512;                // one TMA box: MP tokens x 256 bf16
  static constexpr uint32_t XSLOT = 2 * XBOX;               // a chunk's 512 K
  static constexpr uint32_t SSLOT = kSmTileRows * 8 + kSmTileRows * 8;   // q8 [128][8 B], (d_a, d_b) [128]
  static constexpr uint32_t EROW = MP;                      // floats per row of an epilogue buffer
  static constexpr uint32_t EBUF = 2 * kSmTileRows * EROW * 4;   // [slice][row][token]
  static constexpr uint32_t SUBYTES = MP * 64 * 4;          // sU of one linear as float [t][64]
  static constexpr uint32_t REDBYTES = 128 * 16;            // partial sums of the pieces of X A^T
  static constexpr uint32_t BARBYTES = 128;
  static constexpr uint32_t CRING = kLutBytes;
  static constexpr uint32_t XRING = CRING + NS * kCodeSlot;
  static constexpr uint32_t SRING = XRING + NS * XSLOT;
  static constexpr uint32_t EBUFS = SRING + NS * SSLOT;
  static constexpr uint32_t SUS = EBUFS + 2 * EBUF;
  static constexpr uint32_t REDS = SUS + SUBYTES;
  static constexpr uint32_t BARS = REDS + REDBYTES;
  static constexpr uint32_t END = BARS + BARBYTES + 16;
  static constexpr uint32_t request() { return END; }
};

template <int NT>
__global__ void __launch_bounds__(kSmThreads, 1) nf4_small_m_kernel(const __grid_constant__ SmParams P) {
  constexpr int MP = 8 * NT;
  using L = Layout<MP>;
  constexpr int C = L::C;
  constexpr int NS = L::NS;
  constexpr int D = C / 2;   // own blocks of a consumer warp per chunk
  extern __shared__ __align__(1024) uint8_t smem[];

  if (P.pdl) grid_dep_launch();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;

  const uint32_t base = smem_u32(smem);
  uint8_t *gbase = smem - base;   // generic pointer of shared address 0 (for plain C++ accesses)
  const uint32_t lut = base, cring = base + L::CRING, xring = base + L::XRING, sring = base + L::SRING;
  const uint32_t ebuf = base + L::EBUFS, sus = base + L::SUS, reds = base + L::REDS, bars = base + L::BARS;
  uint64_t *full = reinterpret_cast<uint64_t *>(gbase + bars);
  uint64_t *empty = full + kMaxSlots;
  uint64_t *efull = empty + kMaxSlots;
  uint64_t *eempty = efull + 2;
  volatile int *abort_flag = reinterpret_cast<volatile int *>(gbase + bars + L::BARBYTES);
  int *epi_cmd = reinterpret_cast<int *>(gbase + bars + L::BARBYTES + 4);

  if (L::END > dyn_smem_size()) {   // the host sized this; never expected
    if (threadIdx.x == 0) set_status(P.status, 7 /* QLORA_ERR_CUDA */);
    return;
  }

  // ---- init: the level table, zero activation rows beyond M, barriers ------
  {
    // 16-byte stores: four lanes' copies of one entry at a time
    for (int i = threadIdx.x; i < 2048; i += kSmThreads) {
      const int e = i >> 3, q4 = i & 7;
      const uint32_t lo = __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(kLambda, c_levels[e >> 4])));
      const uint32_t hi = __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(kLambda, c_levels[e & 15])));
      const uint32_t v = lo | (hi << 16);
      *reinterpret_cast<uint4 *>(gbase + lut + e * 256 + q4 * 16) = make_uint4(v, v, v, v);
    }
    if (threadIdx.x == 0) {
      for (int i = 0; i < NS; ++i) {
        mbar_init(&full[i], 1 + 32);   // the producer's expect_tx and its lanes' cp.async arrivals
        mbar_init(&empty[i], kConsumerWarps);
      }
      for (int i = 0; i < 2; ++i) {
        mbar_init(&efull[i], kConsumerWarps);
        mbar_init(&eempty[i], kEpiWarps);
      }
      *abort_flag = 0;
      fence_mbarrier_init();
    }
  }
  __syncthreads();

  const int64_t U = P.w_units, G = gridDim.x;
  const int64_t ub = static_cast<int64_t>(blockIdx.x) * U / G, ue = static_cast<int64_t>(blockIdx.x + 1) * U / G;

  if (warp < kConsumerWarps) {
    // ======================= consumers =======================
    // Warp (rg, slice) owns tile rows 32 rg .. 32 rg + 31 (two 16-row MMA tiles)
    // and the chunk's blocks of parity `slice`.
    const int rg = warp & 3, slice = warp >> 2;
    const uint32_t lreg = static_cast<uint32_t>(lane * 4);
    // code bytes of MMA row g (weight row 2g of a 16-row tile) and row g + 8
    // (weight row 2g + 1): row r of a 128-byte swizzled box holds 16-byte
    // chunk j at 16 (j ^ (r & 7)); this lane reads 8 bytes at byte 8c of block b
    const uint32_t hc = static_cast<uint32_t>(c >> 1), sub = static_cast<uint32_t>(8 * (c & 1));
    uint32_t rbase[2][2], rxor[2][2];
#pragma unroll
    for (int t = 0; t < 2; ++t)
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const uint32_t r = static_cast<uint32_t>(32 * rg + 16 * t + 2 * g + hh);
        rbase[t][hh] = r * 128u + sub;
        rxor[t][hh] = r & 7u;
      }
    float acc[2][NT][4];
#pragma unroll
    for (int t = 0; t < 2; ++t)
#pragma unroll
      for (int u = 0; u < NT; ++u) acc[t][u][0] = acc[t][u][1] = acc[t][u][2] = acc[t][u][3] = 0.f;

    int chunk_idx = 0, seg_idx = 0;
    bool ok = true;
    auto process = [&](const Chunk &cur) {
      const int slot = chunk_idx % NS;
      if (!bar_wait(&full[slot], (chunk_idx / NS) & 1, abort_flag, P.status)) {
        ok = false;
        return;
      }
      const uint32_t cs = cring + slot * kCodeSlot;
      const uint32_t xs = xring + slot * L::XSLOT + g * 512 + 32 * c;
      const int f = cur.kb_s + (((cur.kb_s & 1) != slice) ? 1 : 0);
      const int nown = f < cur.kb_e ? (cur.kb_e - f + 1) / 2 : 0;
      // block scales fp32(q8 * d) / lambda of this lane's four rows (2g, 2g + 1
      // of both tiles) for its own blocks of the chunk; block i of a row uses
      // the first block's second-level constant up to the 256-block group
      // boundary and the last block's after it
      const SmProblem &q = P.p[cur.p];
      float sc[D][4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int row = 32 * rg + 16 * (j >> 1) + 2 * g + (j & 1);
        const uint32_t sq = sring + slot * L::SSLOT + row * 8;
        uint2 q8w, dw;
        asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(q8w.x), "=r"(q8w.y) : "r"(sq));
        asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(dw.x), "=r"(dw.y) : "r"(sq + kSmTileRows * 8));
        const int64_t bi = (static_cast<int64_t>(cur.tile) * kSmTileRows + row) * q.kblocks + cur.kbA;
        const int bnd = 256 - static_cast<int>(bi & 255);
        const float da = __fmul_rn(__uint_as_float(dw.x), kInvLambda), db = __fmul_rn(__uint_as_float(dw.y), kInvLambda);
#pragma unroll
        for (int s = 0; s < D; ++s) {
          const int kbl = f + 2 * s - cur.kbA;
          const uint32_t q8v = prmt(q8w.x, q8w.y, 0x4440u | static_cast<uint32_t>(kbl & 7)) & 0xFFu;
          sc[s][j] = static_cast<float>(q8v) * (kbl < bnd ? da : db);
        }
      }
#pragma unroll
      for (int s = 0; s < D; ++s) {
        if (s < nown) {
          const int kbl = f + 2 * s - cur.kbA;
          const uint32_t half = cs + static_cast<uint32_t>(kbl >> 2) * (kSmTileRows * 128u);
          const uint32_t jj = 2u * static_cast<uint32_t>(kbl & 3) + hc;
          uint2 w[2][2];
#pragma unroll
          for (int t = 0; t < 2; ++t)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              const uint32_t a = half + rbase[t][hh] + 16u * (jj ^ rxor[t][hh]);
              asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(w[t][hh].x), "=r"(w[t][hh].y) : "r"(a));
            }
          uint4 x[NT][2];
          const uint32_t xb = xs + static_cast<uint32_t>(kbl >> 2) * L::XBOX + (kbl & 3) * 128;
#pragma unroll
          for (int u = 0; u < NT; ++u) {
            x[u][0] = lds_u128(xb + u * 8 * 512);
            x[u][1] = lds_u128(xb + u * 8 * 512 + 16);
          }
#pragma unroll
          for (int t = 0; t < 2; ++t) {
            // the four k-steps of the block in two independent chains (steps
            // 0, 2 and 1, 3), added before the block scale
            float tmp[2][NT][4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const uint32_t wa = (i >> 1) ? w[t][0].y : w[t][0].x, wb = (i >> 1) ? w[t][1].y : w[t][1].x;
              const uint32_t sel0 = 0x7604u | ((static_cast<uint32_t>(2 * i) & 3u) << 4);
              const uint32_t sel1 = 0x7604u | ((static_cast<uint32_t>(2 * i + 1) & 3u) << 4);
              const uint32_t a0 = lds_u32(lut + prmt(wa, lreg, sel0));   // MMA row g,     K 4i, 4i+1 of the lane's 16
              const uint32_t a1 = lds_u32(lut + prmt(wb, lreg, sel0));   // MMA row g + 8
              const uint32_t a2 = lds_u32(lut + prmt(wa, lreg, sel1));   // MMA row g,     K 4i+2, 4i+3
              const uint32_t a3 = lds_u32(lut + prmt(wb, lreg, sel1));   // MMA row g + 8
#pragma unroll
              for (int u = 0; u < NT; ++u) {
                const uint32_t b0 = (i == 0) ? x[u][0].x : (i == 1) ? x[u][0].z : (i == 2) ? x[u][1].x : x[u][1].z;
                const uint32_t b1 = (i == 0) ? x[u][0].y : (i == 1) ? x[u][0].w : (i == 2) ? x[u][1].y : x[u][1].w;
                if (i < 2)
                  mma_zero(tmp[i][u], a0, a1, a2, a3, b0, b1);
                else
                  mma_acc(tmp[i & 1][u], a0, a1, a2, a3, b0, b1);
              }
            }
            const float s_lo = sc[s][2 * t], s_hi = sc[s][2 * t + 1];
#pragma unroll
            for (int u = 0; u < NT; ++u) {
              acc[t][u][0] = fmaf(tmp[0][u][0] + tmp[1][u][0], s_lo, acc[t][u][0]);
              acc[t][u][1] = fmaf(tmp[0][u][1] + tmp[1][u][1], s_lo, acc[t][u][1]);
              acc[t][u][2] = fmaf(tmp[0][u][2] + tmp[1][u][2], s_hi, acc[t][u][2]);
              acc[t][u][3] = fmaf(tmp[0][u][3] + tmp[1][u][3], s_hi, acc[t][u][3]);
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[slot]);

      if (cur.last) {   // hand the segment's sums to the epilogue warps
        const int eb = seg_idx & 1;
        if (!bar_wait(&eempty[eb], ((seg_idx >> 1) & 1) ^ 1, abort_flag, P.status)) {
          ok = false;
          return;
        }
        float *dst = reinterpret_cast<float *>(gbase + ebuf + eb * L::EBUF) + slice * kSmTileRows * L::EROW;
#pragma unroll
        for (int t = 0; t < 2; ++t)
#pragma unroll
          for (int u = 0; u < NT; ++u) {
            const int row = 32 * rg + 16 * t + 2 * g;   // weight rows of MMA rows g and g + 8
            *reinterpret_cast<float2 *>(dst + row * L::EROW + 8 * u + 2 * c) = make_float2(acc[t][u][0], acc[t][u][1]);
            *reinterpret_cast<float2 *>(dst + (row + 1) * L::EROW + 8 * u + 2 * c) =
                make_float2(acc[t][u][2], acc[t][u][3]);
            acc[t][u][0] = acc[t][u][1] = acc[t][u][2] = acc[t][u][3] = 0.f;
          }
        __syncwarp();
        if (lane == 0) mbar_arrive(&efull[eb]);
        ++seg_idx;
      }
      ++chunk_idx;
    };

    Walk wk;
    walk_init(wk, ub, ue);
    Chunk cur;
    while (ok && walk_next<C>(P, wk, cur)) process(cur);
  } else if (warp == kProducerWarp) {
    // ======================= producer =======================
    // Per chunk: two TMA boxes of codes and two of activations (lane 0), and
    // each lane's share of the block constants by cp.async: for rows lane,
    // lane + 32, ... the 8 constants of the chunk and the second-level
    // constants of the chunk's first and last block.
    Walk wk;
    walk_init(wk, ub, ue);
    Chunk k;
    int chunk_idx = 0;
    while (walk_next<C>(P, wk, k)) {
      const int slot = chunk_idx % NS;
      if (!bar_wait(&empty[slot], ((chunk_idx / NS) & 1) ^ 1, abort_flag, P.status, 32)) break;
      {
        const SmProblem &q = P.p[k.p];
        const uint32_t sq = sring + slot * L::SSLOT, sd = sq + kSmTileRows * 8;
        const int last = (k.kbA + C < q.kblocks ? k.kbA + C : q.kblocks) - 1;
        const int64_t ngroups = (static_cast<int64_t>(q.N) * q.kblocks + kGroup - 1) / kGroup;
        // 8- or 4-byte copies where every row's 8 constants start aligned
        const uintptr_t a8 = reinterpret_cast<uintptr_t>(q.scale8);
        const bool fast8 = (q.kblocks & 7) == 0 && (a8 & 7) == 0;
        const bool fast4 = (q.kblocks & 3) == 0 && (a8 & 3) == 0;
#pragma unroll
        for (int it = 0; it < 4; ++it) {
          const int row = it * 32 + lane;
          const int64_t n = static_cast<int64_t>(k.tile) * kSmTileRows + row;
          const uint32_t dq = sq + row * 8, dd = sd + row * 8;
          if (n < q.N) {
            const int64_t bi = n * q.kblocks + k.kbA;
            if (fast8) {
              cp_async_8(dq, q.scale8 + bi);
            } else if (fast4) {
              cp_async_4(dq, q.scale8 + bi, 4);
              cp_async_4(dq + 4, q.scale8 + bi + 4, k.kbA + 4 < q.kblocks ? 4 : 0);
            } else {   // rows not 4-byte aligned: plain loads
              uint32_t lo = 0, hi = 0;
              for (int i = 0; i < 8; ++i)
                if (k.kbA + i < q.kblocks) {
                  const uint32_t v = static_cast<uint32_t>(__ldg(q.scale8 + bi + i));
                  if (i < 4) lo |= v << (8 * i); else hi |= v << (8 * (i - 4));
                }
              *reinterpret_cast<uint2 *>(gbase + dq) = make_uint2(lo, hi);
            }
            const int64_t ga = bi >> 8, gb = (n * q.kblocks + last) >> 8;
            cp_async_4(dd, q.scale2 + ga, 4);
            cp_async_4(dd + 4, q.scale2 + (gb < ngroups ? gb : ga), 4);
          }
        }
        if (fast4) {
          cp_async_arrive(&full[slot]);
        } else {   // plain stores above: complete the copies, then a releasing arrival
          asm volatile("cp.async.wait_all;" ::: "memory");
          mbar_arrive(&full[slot]);
        }
      }
      if (lane == 0) {
        const SmProblem &q = P.p[k.p];
        const int nblk = (k.kbA + C < q.kblocks ? k.kbA + C : q.kblocks) - k.kbA;
        const uint32_t cdst = cring + slot * kCodeSlot, xdst = xring + slot * L::XSLOT;
        uint32_t tx = kSmTileRows * 128u + L::XBOX;
        if (chunk_idx == 0 && P.pdl) grid_dep_wait();   // activations may come from the preceding launch
        tma_load_2d(gbase + cdst, &P.tm_codes[k.p], &full[slot], k.kbA * 32, k.tile * kSmTileRows);
        tma_load_2d(gbase + xdst, &P.tm_x[k.p], &full[slot], k.kbA * 64, 0);
        if (nblk > 4) {
          tma_load_2d(gbase + cdst + kSmTileRows * 128u, &P.tm_codes[k.p], &full[slot], k.kbA * 32 + 128,
                      k.tile * kSmTileRows);
          tma_load_2d(gbase + xdst + L::XBOX, &P.tm_x[k.p], &full[slot], k.kbA * 64 + 256, 0);
          tx += kSmTileRows * 128u + L::XBOX;
        }
        mbar_arrive_expect_tx(&full[slot], tx);
      }
      __syncwarp();
      ++chunk_idx;
    }
    // do not leave while copies into this CTA's shared memory may be in flight
    if (*abort_flag && chunk_idx > 0) {
      for (int i = chunk_idx - 1; i >= 0 && i >= chunk_idx - NS; --i) {
        const uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait(&full[i % NS], (i / NS) & 1) && global_timer_ns() - t0 < kWaitLimitNs) {
        }
      }
    }
  } else {
    // ======================= epilogue =======================
    const int et = threadIdx.x - kEpiWarp0 * 32;   // 0..127: a tile row
    const int ew = et >> 5;
    if (P.pdl) grid_dep_wait();

    // ---- pieces of X A^T: 128 K each, every load issued before the MMAs ----
    // Inside each 64-K block the K order is permuted as in the weight path: lane
    // (g, c) holds K 16c .. 16c + 15 of a row, so its fragments are two 16-byte
    // loads per row and block.
    for (int64_t qi = static_cast<int64_t>(blockIdx.x) * kEpiWarps + ew; qi < P.u_units;
         qi += static_cast<int64_t>(gridDim.x) * kEpiWarps) {
      int p = 0;
      for (int i = 1; i < P.count; ++i)
        if (qi >= P.p[i].u_unit0 && P.p[i].A) p = i;
      const SmProblem &q = P.p[p];
      const int ch = static_cast<int>(qi - q.u_unit0);
      const int k0 = ch * kUnitK;
      const bool two = k0 + 64 < q.K;   // the last piece may hold one block
      const int r16 = (q.r + 15) / 16;
      uint4 xv[2][NT][2];
#pragma unroll
      for (int bl = 0; bl < 2; ++bl)
#pragma unroll
        for (int u = 0; u < NT; ++u) {
          const int t = 8 * u + g;
          const uint4 *xr = reinterpret_cast<const uint4 *>(q.X + static_cast<int64_t>(t) * q.K + k0 + 64 * bl + 16 * c);
          const bool ok = t < P.M && (bl == 0 || two);
          xv[bl][u][0] = ok ? __ldg(xr) : make_uint4(0, 0, 0, 0);
          xv[bl][u][1] = ok ? __ldg(xr + 1) : make_uint4(0, 0, 0, 0);
        }
      float d[4][NT][4];
#pragma unroll
      for (int jt = 0; jt < 4; ++jt) {
#pragma unroll
        for (int u = 0; u < NT; ++u) d[jt][u][0] = d[jt][u][1] = d[jt][u][2] = d[jt][u][3] = 0.f;
        if (jt < r16) {
          uint4 av[2][2][2];   // [block][row g / g + 8][half]
#pragma unroll
          for (int bl = 0; bl < 2; ++bl)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int j = 16 * jt + g + 8 * h;
              const uint4 *ar = reinterpret_cast<const uint4 *>(q.A + static_cast<int64_t>(j) * q.K + k0 + 64 * bl + 16 * c);
              const bool ok = j < q.r && (bl == 0 || two);
              av[bl][h][0] = ok ? __ldg(ar) : make_uint4(0, 0, 0, 0);
              av[bl][h][1] = ok ? __ldg(ar + 1) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
          for (int bl = 0; bl < 2; ++bl)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const uint4 &ag = av[bl][0][i >> 1], &ah = av[bl][1][i >> 1];
              const uint32_t a0 = (i & 1) ? ag.z : ag.x, a2 = (i & 1) ? ag.w : ag.y;
              const uint32_t a1 = (i & 1) ? ah.z : ah.x, a3 = (i & 1) ? ah.w : ah.y;
#pragma unroll
              for (int u = 0; u < NT; ++u) {
                const uint4 &xx = xv[bl][u][i >> 1];
                mma_acc(d[jt][u], a0, a1, a2, a3, (i & 1) ? xx.z : xx.x, (i & 1) ? xx.w : xx.y);
              }
            }
        }
      }
      float *up = q.upart + static_cast<int64_t>(ch) * (16 * r16) * MP;
#pragma unroll
      for (int jt = 0; jt < 4; ++jt)
        if (jt < r16)
#pragma unroll
          for (int u = 0; u < NT; ++u) {
            const int j = 16 * jt + g, t = 8 * u + 2 * c;
            *reinterpret_cast<float2 *>(up + j * MP + t) = make_float2(d[jt][u][0], d[jt][u][1]);
            *reinterpret_cast<float2 *>(up + (j + 8) * MP + t) = make_float2(d[jt][u][2], d[jt][u][3]);
          }
      __syncwarp();
      if (lane == 0) {
        __threadfence();   // after the warp barrier: covers the whole warp's partial sums
        atomicAdd(&P.ucnt[p], 1ull);
      }
    }

    // ---- finished segments ----
    float *su_s = reinterpret_cast<float *>(gbase + sus);
    int su_p = -1;   // the linear whose sU su_s holds
    Walk wk;
    walk_init(wk, ub, ue);
    Chunk k;
    int seg_idx = 0;
    const int64_t self = blockIdx.x;
    while (walk_next<C>(P, wk, k)) {
      if (!k.last) continue;
      const int eb = seg_idx & 1;
      if (!bar_wait(&efull[eb], (seg_idx >> 1) & 1, abort_flag, P.status, 64)) break;
      const float *src = reinterpret_cast<const float *>(gbase + ebuf + eb * L::EBUF);
      float sum[MP];
#pragma unroll
      for (int t = 0; t < MP; t += 4) {
        const float4 a = *reinterpret_cast<const float4 *>(src + et * L::EROW + t);
        const float4 b = *reinterpret_cast<const float4 *>(src + (kSmTileRows + et) * L::EROW + t);
        sum[t] = a.x + b.x;
        sum[t + 1] = a.y + b.y;
        sum[t + 2] = a.z + b.z;
        sum[t + 3] = a.w + b.w;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&eempty[eb]);
      ++seg_idx;

      const SmProblem &q = P.p[k.p];
      const int64_t n = static_cast<int64_t>(k.tile) * kSmTileRows + et;
      const bool tile_first = k.seg_lo == 0, tile_last = k.seg_hi == q.kblocks;
      if (!tile_first) {
        // a later contributor: publish the partial for the CTA holding the tile's first block
        float *slot = P.slots + self * (MP * kSmTileRows);
#pragma unroll
        for (int t = 0; t < MP; ++t)
          if (t < P.M) slot[t * kSmTileRows + et] = sum[t];
        // the barrier orders every thread's stores before thread 0's release,
        // which is cumulative: the flag publishes all of them at GPU scope
        named_barrier(kEpiBar, kEpiWarps * 32);
        if (et == 0) {
          __threadfence();
          st_release_gpu_u64(&P.flags[self], P.epoch);
        }
        continue;
      }
      if (!tile_last) {
        // owner of a split tile: add the later contributors' partials in CTA order
        const int64_t last_unit = q.w_unit0 + static_cast<int64_t>(k.tile + 1) * q.kblocks - 1;
        const int b1 = cta_of(last_unit, P.w_units, gridDim.x);
        // thread i waits for contributor self + 1 + i (all at once), then the
        // partials are added in CTA order
        if (et == 0) epi_cmd[0] = 1;
        named_barrier(kEpiBar, kEpiWarps * 32);
        for (int bb = static_cast<int>(self) + 1 + et; bb <= b1; bb += kEpiWarps * 32)
          if (!wait_word(&P.flags[bb], P.epoch, abort_flag, P.status)) epi_cmd[0] = 0;
        named_barrier(kEpiBar, kEpiWarps * 32);
        const bool ok = epi_cmd[0] != 0;
        named_barrier(kEpiBar, kEpiWarps * 32);
        if (!ok) break;
        for (int bb = static_cast<int>(self) + 1; bb <= b1; ++bb) {
          const float *slot = P.slots + static_cast<int64_t>(bb) * (MP * kSmTileRows);
#pragma unroll
          for (int t = 0; t < MP; ++t)
            if (t < P.M) sum[t] += __ldcg(slot + t * kSmTileRows + et);
        }
        named_barrier(kEpiBar, kEpiWarps * 32);
        if (et == 0)
          for (int bb = static_cast<int>(self) + 1; bb <= b1; ++bb) P.flags[bb] = 0;
      }
      // finish the tile: the LoRA term in fp32, then Y in bf16
      if (k.p != su_p) {   // sU of this linear, once per CTA
        if (q.sU_in != nullptr) {
          for (int i = et; i < P.M * q.r; i += kEpiWarps * 32) {
            const int t = i / q.r, j = i % q.r;
            su_s[t * 64 + j] = __uint_as_float(static_cast<uint32_t>(__ldg(q.sU_in + i)) << 16);
          }
        } else {
          // wait for every piece of X A^T, then add them in a fixed order:
          // thread (part, col) sums pieces part, part + nsplit, ... of float4
          // column col; the parts are then added in order
          if (et == 0)
            epi_cmd[0] = wait_word(reinterpret_cast<const uint64_t *>(&P.ucnt[k.p]),
                                   static_cast<uint64_t>(q.uchunks), abort_flag, P.status) ? 1 : 0;
          named_barrier(kEpiBar, kEpiWarps * 32);
          if (epi_cmd[0] == 0) break;
          const int r16 = (q.r + 15) / 16;
          const int cols = 16 * r16 * MP / 4;                 // float4 columns of one piece
          const int nsplit = cols >= 128 ? 1 : 128 / cols;    // 1, 2 or 4 (cols is 32, 64, 128 ...)
          float4 *red4 = reinterpret_cast<float4 *>(gbase + reds);
          for (int col0 = 0; col0 < cols; col0 += 128 / nsplit) {
            const int col = col0 + et % (128 / nsplit), part = et / (128 / nsplit);
            float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
            if (col < cols) {
              const float4 *src4 = reinterpret_cast<const float4 *>(q.upart) + col;
              int cc = part;
              for (; cc + 3 * nsplit < q.uchunks; cc += 4 * nsplit) {
                const float4 v0 = __ldcg(src4 + static_cast<int64_t>(cc) * cols);
                const float4 v1 = __ldcg(src4 + static_cast<int64_t>(cc + nsplit) * cols);
                const float4 v2 = __ldcg(src4 + static_cast<int64_t>(cc + 2 * nsplit) * cols);
                const float4 v3 = __ldcg(src4 + static_cast<int64_t>(cc + 3 * nsplit) * cols);
                a.x += v0.x; a.y += v0.y; a.z += v0.z; a.w += v0.w;
                a.x += v1.x; a.y += v1.y; a.z += v1.z; a.w += v1.w;
                a.x += v2.x; a.y += v2.y; a.z += v2.z; a.w += v2.w;
                a.x += v3.x; a.y += v3.y; a.z += v3.z; a.w += v3.w;
              }
              for (; cc < q.uchunks; cc += nsplit) {
                const float4 v = __ldcg(src4 + static_cast<int64_t>(cc) * cols);
                a.x += v.x; a.y += v.y; a.z += v.z; a.w += v.w;
              }
            }
            red4[et] = a;
            named_barrier(kEpiBar, kEpiWarps * 32);
            if (part == 0 && col < cols) {
              float4 t4 = red4[et];
              for (int pp = 1; pp < nsplit; ++pp) {
                const float4 v = red4[et + pp * (128 / nsplit)];
                t4.x += v.x; t4.y += v.y; t4.z += v.z; t4.w += v.w;
              }
              // column col holds U[j][t .. t + 3] with j = 4 col / MP, t = 4 col % MP
              const int j = (4 * col) / MP, t0 = (4 * col) % MP;
              const float uv[4] = {t4.x, t4.y, t4.z, t4.w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const int t = t0 + e;
                if (j < q.r && t < P.M) {
                  const __nv_bfloat16 b = __float2bfloat16_rn(q.s * uv[e]);
                  su_s[t * 64 + j] = __bfloat162float(b);
                  if (k.tile == 0) q.sU[static_cast<int64_t>(t) * q.r + j] = __bfloat16_as_ushort(b);
                }
              }
            }
            named_barrier(kEpiBar, kEpiWarps * 32);
          }
        }
        su_p = k.p;
      }
      named_barrier(kEpiBar, kEpiWarps * 32);
      if (n < q.N) {
        float y[MP];
#pragma unroll
        for (int t = 0; t < MP; ++t) y[t] = sum[t];
        const uint4 *brow = reinterpret_cast<const uint4 *>(q.B + n * q.r);
        for (int j8 = 0; j8 < q.r / 8; ++j8) {
          const uint4 bv = __ldg(brow + j8);
          const uint32_t bw[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
          for (int h = 0; h < 8; ++h) {
            const float bj = __uint_as_float((h & 1) ? (bw[h >> 1] & 0xFFFF0000u) : (bw[h >> 1] << 16));
#pragma unroll
            for (int t = 0; t < MP; ++t) y[t] = fmaf(su_s[t * 64 + 8 * j8 + h], bj, y[t]);
          }
        }
#pragma unroll
        for (int t = 0; t < MP; ++t)
          if (t < P.M) q.Y[static_cast<int64_t>(t) * q.N + n] = __bfloat16_as_ushort(__float2bfloat16_rn(y[t]));
      }
      named_barrier(kEpiBar, kEpiWarps * 32);
      if (q.sU_in == nullptr && et == 0) {
        if (atomicAdd(&P.ucons[k.p], 1ull) + 1 == static_cast<unsigned long long>(q.tiles)) {   // the last user
          atomicExch(&P.ucnt[k.p], 0ull);
          atomicExch(&P.ucons[k.p], 0ull);
        }
      }
    }
  }
}

// ---- host side -----------------------------------------------------------------
uint64_t next_epoch() {
  static std::atomic<uint64_t> counter{static_cast<uint64_t>(
      std::chrono::steady_clock::now().time_since_epoch().count()) * 0x9E3779B97F4A7C15ull};
  const uint64_t v = counter.fetch_add(1, std::memory_order_relaxed);
  return v % ((1ull << 44) - 1) + 1;
}

size_t up256(size_t x) { return (x + 255) / 256 * 256; }

struct SmWsLayout {
  size_t flags, slots, total;
  size_t upart[kSmMaxProblems], su[kSmMaxProblems];
};

SmWsLayout sm_ws_layout(const SmallProblem *pr, int count, int64_t M) {
  SmWsLayout w{};
  const size_t G = static_cast<size_t>(device_sm_count());
  const int MP = M <= 8 ? 8 : 16;
  size_t off = 0;
  w.flags = off;
  off += up256(G * 8);
  w.slots = off;
  off += up256(G * MP * kSmTileRows * 4);
  for (int i = 0; i < count; ++i) {
    w.upart[i] = w.su[i] = 0;
    if (pr[i].A) {
      const size_t uch = static_cast<size_t>((pr[i].K + kUnitK - 1) / kUnitK);
      const size_t r16 = static_cast<size_t>((pr[i].r + 15) / 16);
      w.upart[i] = off;
      off += up256(uch * 16 * r16 * MP * 4);
      if (!pr[i].sU_out) {
        w.su[i] = off;
        off += up256(static_cast<size_t>(M) * pr[i].r * 2);
      }
    }
  }
  w.total = off;
  return w;
}

}  // namespace

size_t small_m_ws_bytes(const SmallProblem *pr, int count, int64_t M) {
  size_t total = 0;
  for (int i0 = 0; i0 < count; i0 += kSmMaxProblems) {
    const int n = count - i0 < kSmMaxProblems ? count - i0 : kSmMaxProblems;
    const size_t t = sm_ws_layout(pr + i0, n, M).total;
    total = t > total ? t : total;
  }
  return total;
}

int small_m_max_problems() { return kSmMaxProblems; }

cudaError_t launch_small_m(const SmallProblem *pr, int count, int64_t M, void *ws, void *counters, bool pdl,
                           int32_t *status, cudaStream_t st) {
  for (int i0 = 0; i0 < count; i0 += kSmMaxProblems) {
    const int n = count - i0 < kSmMaxProblems ? count - i0 : kSmMaxProblems;
    const SmallProblem *q = pr + i0;
    const SmWsLayout w = sm_ws_layout(q, n, M);
    uint8_t *wsb = static_cast<uint8_t *>(ws);
    SmParams P{};
    P.count = n;
    P.M = static_cast<int32_t>(M);
    int64_t wu = 0;
    int32_t uu = 0;
    for (int i = 0; i < n; ++i) {
      if (!encode_2d(&P.tm_codes[i], CU_TENSOR_MAP_DATA_TYPE_UINT8, q[i].codes, static_cast<uint64_t>(q[i].K / 2),
                     static_cast<uint64_t>(q[i].N), static_cast<uint64_t>(q[i].K / 2), 128, kSmTileRows,
                     CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
      if (!encode_2d(&P.tm_x[i], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, q[i].X, static_cast<uint64_t>(q[i].K),
                     static_cast<uint64_t>(M), static_cast<uint64_t>(q[i].K) * 2, 256, M > 8 ? 16 : 8,
                     CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
      SmProblem &p = P.p[i];
      p.codes = q[i].codes;
      p.scale8 = q[i].scale8;
      p.scale2 = q[i].scale2;
      p.X = q[i].X;
      p.A = q[i].A;
      p.B = q[i].B;
      p.sU_in = q[i].sU_in;
      p.Y = q[i].Y;
      p.N = static_cast<int32_t>(q[i].N);
      p.K = static_cast<int32_t>(q[i].K);
      p.kblocks = p.K / kBlock;
      p.tiles = (p.N + kSmTileRows - 1) / kSmTileRows;
      p.r = q[i].r;
      p.s = q[i].s;
      p.w_unit0 = wu;
      wu += static_cast<int64_t>(p.tiles) * p.kblocks;
      p.u_unit0 = uu;
      if (q[i].A) {
        p.uchunks = (p.K + kUnitK - 1) / kUnitK;
        p.upart = reinterpret_cast<float *>(wsb + w.upart[i]);
        p.sU = q[i].sU_out ? q[i].sU_out : reinterpret_cast<uint16_t *>(wsb + w.su[i]);
        uu += p.uchunks;
      } else {
        p.uchunks = 0;
        p.upart = nullptr;
        p.sU = nullptr;
      }
    }
    P.w_units = wu;
    P.u_units = uu;
    P.epoch = next_epoch();
    P.flags = reinterpret_cast<uint64_t *>(wsb + w.flags);
    P.ucnt = static_cast<unsigned long long *>(counters);
    P.ucons = P.ucnt + kSmMaxProblems;
    P.slots = reinterpret_cast<float *>(wsb + w.slots);
    P.status = status;
    P.pdl = pdl ? 1 : 0;

    const int sms = device_sm_count();
    const int grid = static_cast<int>(wu < sms ? wu : sms);
    const bool nt2 = M > 8;
    const void *fn = nt2 ? reinterpret_cast<const void *>(nf4_small_m_kernel<2>)
                         : reinterpret_cast<const void *>(nf4_small_m_kernel<1>);
    const uint32_t smem = nt2 ? Layout<16>::request() : Layout<8>::request();
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(kSmThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    void *args[] = {&P};
    e = cudaLaunchKernelExC(&cfg, fn, args);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace qlora
