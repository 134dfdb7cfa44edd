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
//   warp holds loads in flight in its registers.
// * Two scale warps bring the chunk's 8-bit block constants and its
//   second-level constants into a ring of their own (a TMA copy of each, or
//   cp.async where K does not suit the copy's 16-byte rule), form the fp32
//   block scales of all 128 rows and publish them in a third ring, laid out
//   in the order the consumer lanes read them.
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
//   epilogue warps of all CTAs split X A^T into 128-K pieces, the last piece
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
#include <cstring>

#include "qlora_device.cuh"

namespace qlora {

bool encode_2d(CUtensorMap *map, CUtensorMapDataType dtype, const void *base, uint64_t inner, uint64_t outer,
               uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swizzle);
bool encode_3d(CUtensorMap *map, CUtensorMapDataType dtype, const void *base, const uint64_t dims[3],
               const uint64_t strides[2], const uint32_t box[3], CUtensorMapSwizzle swizzle);

namespace {

constexpr int kSmMaxProblems = 16;                  // linears per launch (the counter page holds 2 x 16 counters)
constexpr int kSmTileRows = 128;
constexpr int kConsumerWarps = 8;                    // 4 row groups x 2 K slices
constexpr int kProducerWarp = 8;                     // the copies of codes and activations
constexpr int kScaleWarp0 = 9;                       // the block scales: rows 0-63 and 64-127
constexpr int kScaleWarps = 2;
constexpr int kEpiWarp0 = kScaleWarp0 + kScaleWarps;
constexpr int kEpiWarps = 4;
constexpr int kSmThreads = (kEpiWarp0 + kEpiWarps) * 32;   // 480
constexpr int kChunkBlocks = 8;                      // NF4 blocks (of 64 weights) per chunk
constexpr uint32_t kCodeSlot = kSmTileRows * kChunkBlocks * 32;   // 32 KB of codes per chunk
constexpr int kUnitK = 128;                          // K per piece of X A^T (two NF4 blocks)
constexpr uint32_t kLutBytes = 65536;                // 256 entries x 256 B (32 lanes x 4 B + unused half)
constexpr int kMaxSlots = 3;
constexpr float kLambda = 1.43675f;
constexpr float kInvLambda = 1.0f / 1.43675f;
constexpr uint32_t kEpiBar = 1;                      // named barrier of the epilogue warps
constexpr uint32_t kTableBar = 2;                    // named barrier of the consumer warps

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

// What the kernel reads besides the tensor maps; copied into shared memory
// at the start of a launch by all threads at once (one round of parameter
// loads instead of a chain of dependent ones).
struct __align__(16) SmHead {
  SmProblem p[kSmMaxProblems];
  int32_t count, M;
  int64_t w_units;
  int32_t u_units;
  int32_t pdl;
  int32_t x3d;             // tm_x is the 3-D map (one box per chunk), else one 2-D box per block
  int32_t rawtma;          // raw constants by TMA (tm_q8, tm_s2), else by cp.async
  int32_t pad_[2];
  uint64_t epoch;          // launch value, 1 <= epoch < 2^44
  uint64_t *flags;         // [grid]: a contributor's partial is published; then [count]: sU ready
  float *slots;            // [grid][MP][128]: published partials
  unsigned long long *ucnt;    // [count]: pieces of X A^T done (zero at launch)
  unsigned long long *ucons;   // [count]: tiles that have used them (zero at launch)
  int32_t *status;
  uint16_t lvl[16];        // bf16(lambda * level[i])
};
static_assert(sizeof(SmHead) % 16 == 0, "copied as 16-byte words");
static_assert(2 * kSmMaxProblems * 8 <= kSmallCounterBytes, "ucnt and ucons fit the counter page");

struct SmParams {
  CUtensorMap tm_codes[kSmMaxProblems];   // codes of each linear as u8 [N][K/2], 128 x 128-byte boxes, swizzled
  CUtensorMap tm_x[kSmMaxProblems];       // activations as bf16 [M][K]: boxes [8 blocks][MP tokens][64], swizzled
  CUtensorMap tm_q8[kSmMaxProblems];      // first-level constants as u8 [N][K/64], boxes 16 x 128
  CUtensorMap tm_s2[kSmMaxProblems];      // second-level constants as f32 [1][groups], boxes of 256
  SmHead h;
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
__device__ __forceinline__ int problem_of(const SmHead &P, int64_t u) {
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
__device__ __forceinline__ bool walk_next(const SmHead &P, Walk &w, Chunk &c) {
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
// The level table sits at a 64 KB-aligned shared address, so that one PRMT
// forms a lookup's whole address (table | byte << 8 | lane * 4). Its entries
// use the first 128 bytes of every 256; the second halves hold the epilogue
// buffers (byte o of them at lut + 256 (o >> 7) + 128 + (o & 127)). The space
// between the start of dynamic shared memory and the table takes the rings of
// activations, block scales and raw constants, sU and the barriers, or, if
// they do not fit there, goes after the code ring.
template <int MP>
struct Layout {
  static constexpr int C = kChunkBlocks;
  static constexpr int NS = MP == 8 ? 3 : 2;                // ring depth
  static constexpr uint32_t XBOX = MP * 128;                // a block of MP tokens: [token][64 bf16], 128-byte swizzle
  static constexpr uint32_t XSLOT = C * XBOX;               // a chunk's 512 K
  static constexpr uint32_t SCSLOT = C * kSmTileRows * 4;   // block scales [block][row group][g][4] floats
  static constexpr uint32_t RAWQ8 = kSmTileRows * 16;       // raw q8: [row][16 B], the chunk's 8 at byte kbA % 16
  static constexpr uint32_t RAWSLOT = RAWQ8 + 1024;         // then 256 second-level constants, or (d_a, d_b) per row
  static constexpr uint32_t EROW = MP;                      // floats per row of an epilogue buffer
  static constexpr uint32_t EBUF = 2 * kSmTileRows * EROW * 4;   // [slice][row][token]
  static_assert(2 * EBUF <= kLutBytes / 2, "epilogue buffers fit the table's second halves");
  static constexpr uint32_t SUBYTES = MP * 64 * 4;          // sU of one linear as float [t][64]
  static constexpr uint32_t BARBYTES = 256;
  static constexpr uint32_t S_X = 0;
  static constexpr uint32_t S_SC = S_X + NS * XSLOT;
  static constexpr uint32_t S_RAW = S_SC + NS * SCSLOT;
  static constexpr uint32_t S_SU = S_RAW + NS * RAWSLOT;
  static constexpr uint32_t S_HEAD = S_SU + SUBYTES;        // the launch's head (parameters)
  static constexpr uint32_t S_BAR = S_HEAD + static_cast<uint32_t>(sizeof(SmHead));
  static constexpr uint32_t G1 = S_BAR + BARBYTES + 16;
  static constexpr uint32_t CODES = NS * kCodeSlot;
  // bytes used from the start of dynamic shared memory at shared address
  // `base`; the small regions start on a 1 KB boundary (swizzled TMA boxes)
  static constexpr uint32_t extent(uint32_t base) {
    const uint32_t lut = (base + 0xFFFFu) & ~0xFFFFu, avail = lut - ((base + 1023u) & ~1023u);
    return lut - base + kLutBytes + CODES + (G1 <= avail ? 0 : G1);
  }
  // dynamic shared memory to request: the largest extent over the starts
  // this kernel can see (16-byte aligned, at most 4 KB)
  static constexpr uint32_t request() {
    uint32_t m = 0;
    for (uint32_t b = 0; b <= 4096; b += 16) m = extent(b) > m ? extent(b) : m;
    return m;
  }
};
static_assert(Layout<8>::request() <= 232448 && Layout<16>::request() <= 232448, "shared memory");

template <int NT>
__global__ void __launch_bounds__(kSmThreads, 1) nf4_small_m_kernel(const __grid_constant__ SmParams Pk) {
  constexpr int MP = 8 * NT;
  using L = Layout<MP>;
  constexpr int C = L::C;
  constexpr int NS = L::NS;
  constexpr int D = C / 2;   // own blocks of a consumer warp per chunk
  extern __shared__ __align__(1024) uint8_t smem[];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;

  // ---- layout --------------------------------------------------------------
  const uint32_t base = smem_u32(smem);
  uint8_t *gbase = smem - base;   // generic pointer of shared address 0 (for plain C++ accesses)
  const uint32_t lut = (base + 0xFFFFu) & ~0xFFFFu;
  const uint32_t cring = lut + kLutBytes;
  const uint32_t low = (base + 1023u) & ~1023u;
  const uint32_t g1 = L::G1 <= lut - low ? low : cring + L::CODES;
  // byte o of the epilogue buffers
  auto egap = [lut](uint32_t o) { return lut + ((o >> 7) << 8) + 128u + (o & 127u); };
  const uint32_t xring = g1 + L::S_X, scring = g1 + L::S_SC, rawring = g1 + L::S_RAW;
  const uint32_t sus = g1 + L::S_SU, bars = g1 + L::S_BAR;
  SmHead &s_head = *reinterpret_cast<SmHead *>(gbase + g1 + L::S_HEAD);
  const SmHead &P = s_head;
  const uint32_t end = base + L::extent(base);
  uint64_t *full = reinterpret_cast<uint64_t *>(gbase + bars);
  uint64_t *sfull = full + kMaxSlots;
  uint64_t *empty = sfull + kMaxSlots;
  uint64_t *rfull = empty + kMaxSlots;   // raw constants by TMA
  uint64_t *efull = rfull + kMaxSlots;
  uint64_t *eempty = efull + 2;
  volatile int *abort_flag = reinterpret_cast<volatile int *>(gbase + bars + L::BARBYTES);
  int *epi_cmd = reinterpret_cast<int *>(gbase + bars + L::BARBYTES + 4);

  if (end > base + dyn_smem_size()) {   // the host sized this; never expected
    if (threadIdx.x == 0) set_status(Pk.h.status, 7 /* QLORA_ERR_CUDA */);
    return;
  }

  {
    const uint4 *src = reinterpret_cast<const uint4 *>(&Pk.h);
    uint4 *dst = reinterpret_cast<uint4 *>(&s_head);
    for (int i = threadIdx.x; i < static_cast<int>(sizeof(SmHead) / 16); i += kSmThreads) dst[i] = src[i];
  }
  if (warp == kProducerWarp) {   // the descriptors of this launch's copies
    const int cnt = Pk.h.count;
    if (lane < cnt) prefetch_tensormap(&Pk.tm_codes[lane]);
    if (lane >= 16 && lane - 16 < cnt) prefetch_tensormap(&Pk.tm_x[lane - 16]);
  }
  if (threadIdx.x == 0) {
    for (int i = 0; i < NS; ++i) {
      mbar_init(&full[i], 1);   // the producer's arrival with the copies' bytes
      mbar_init(&sfull[i], kScaleWarps);
      mbar_init(&empty[i], kConsumerWarps);
      mbar_init(&rfull[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&efull[i], kConsumerWarps);
      mbar_init(&eempty[i], kEpiWarps);
    }
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  __syncthreads();
  if (P.pdl) grid_dep_launch();

  const int64_t U = P.w_units, G = gridDim.x;
  const int64_t ub = static_cast<int64_t>(blockIdx.x) * U / G, ue = static_cast<int64_t>(blockIdx.x + 1) * U / G;

  // ---- producer pieces ------------------------------------------------------
  const int sw = warp - kScaleWarp0;   // a scale warp's half of the tile rows
  // Raw constants of a chunk by cp.async into raw slot rs (one commit group):
  // for rows lane, lane + 32, ... the chunk's 8 q8 bytes and the second-level
  // constants of its first and last block.
  auto issue_raw = [&](const Chunk &k, int rs) {
    const SmProblem &q = P.p[k.p];
    const uint32_t sq = rawring + rs * L::RAWSLOT, sd = sq + L::RAWQ8;
    const int last = (k.kbA + C < q.kblocks ? k.kbA + C : q.kblocks) - 1;
    const int64_t ngroups = (static_cast<int64_t>(q.N) * q.kblocks + kGroup - 1) / kGroup;
    const uintptr_t a8 = reinterpret_cast<uintptr_t>(q.scale8);
    const bool fast8 = (q.kblocks & 7) == 0 && (a8 & 7) == 0;
    const bool fast4 = (q.kblocks & 3) == 0 && (a8 & 3) == 0;
#pragma unroll
    for (int it = 2 * sw; it < 2 * sw + 2; ++it) {
      const int row = it * 32 + lane;
      const int64_t n = static_cast<int64_t>(k.tile) * kSmTileRows + row;
      const uint32_t dq = sq + row * 16 + (k.kbA & 15), dd = sd + row * 8;
      if (n < q.N) {
        const int64_t bi = n * q.kblocks + k.kbA;
        if (fast8) {
          cp_async_8(dq, q.scale8 + bi);
        } else if (fast4) {
          cp_async_4(dq, q.scale8 + bi, 4);
          cp_async_4(dq + 4, q.scale8 + bi + 4, k.kbA + 4 < q.kblocks ? 4 : 0);
        } else {   // rows not 4-byte aligned: plain loads (ordered by the wait before use)
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
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  // Codes (two 128-row boxes of four blocks) and activations of a chunk into
  // ring slot `slot`, counted on full[slot]; one thread.
  auto issue_tma = [&](const Chunk &k, int slot, int chunk_idx) {
    const SmProblem &q = P.p[k.p];
    const int nblk = (k.kbA + C < q.kblocks ? k.kbA + C : q.kblocks) - k.kbA;
    const uint32_t cdst = cring + slot * kCodeSlot, xdst = xring + slot * L::XSLOT;
    const uint32_t xbytes = (P.x3d ? C : nblk) * L::XBOX;   // a 3-D box counts its zero-filled blocks too
    mbar_arrive_expect_tx(&full[slot], (nblk > 4 ? 2u : 1u) * (kSmTileRows * 128u) + xbytes);
    // codes are read once per launch: they should not push the activations,
    // adapters and partial sums out of L2
    const uint64_t pol = l2_evict_first_policy();
    tma_load_2d_hint(gbase + cdst, &Pk.tm_codes[k.p], &full[slot], k.kbA * 32, k.tile * kSmTileRows, pol);
    if (nblk > 4)
      tma_load_2d_hint(gbase + cdst + kSmTileRows * 128u, &Pk.tm_codes[k.p], &full[slot], k.kbA * 32 + 128,
                       k.tile * kSmTileRows, pol);
    if (chunk_idx == 0 && P.pdl) grid_dep_wait();   // activations may come from the preceding launch
    if (P.x3d)
      tma_load_3d(gbase + xdst, &Pk.tm_x[k.p], &full[slot], 0, 0, k.kbA);
    else
      for (int b = 0; b < nblk; ++b)
        tma_load_2d(gbase + xdst + b * L::XBOX, &Pk.tm_x[k.p], &full[slot], (k.kbA + b) * 64, 0);
  };
  // Raw constants of a chunk by TMA into raw slot `slot`, counted on
  // rfull[slot]: the 16-byte column of q8 holding the chunk's 8 blocks for
  // 128 rows, and 256 second-level constants from the (4-aligned) group of
  // the tile's first row; one thread.
  auto issue_raw_tma = [&](const Chunk &k, int slot) {
    const SmProblem &q = P.p[k.p];
    const uint32_t sq = rawring + slot * L::RAWSLOT;
    const int64_t bi0 = static_cast<int64_t>(k.tile) * kSmTileRows * q.kblocks + k.kbA;
    mbar_arrive_expect_tx(&rfull[slot], L::RAWSLOT);
    tma_load_2d(gbase + sq, &Pk.tm_q8[k.p], &rfull[slot], k.kbA & ~15, k.tile * kSmTileRows);
    tma_load_2d(gbase + sq + L::RAWQ8, &Pk.tm_s2[k.p], &rfull[slot], static_cast<int32_t>((bi0 >> 8) & ~int64_t{3}), 0);
  };
  // Block scales of a chunk from its raw constants: s = q8 * (d / lambda),
  // stored [block][row group][g][h] with h = 2 t + hh for weight row
  // 32 rg + 16 t + 2 g + hh (the rows of a consumer lane); then one arrival
  // on sfull[slot].
  auto publish_scales = [&](const Chunk &k, int slot) {
    const SmProblem &q = P.p[k.p];
    const uint32_t sq = rawring + slot * L::RAWSLOT, sd = sq + L::RAWQ8;
    const float *s2w = reinterpret_cast<const float *>(gbase + sd);
    float *scs = reinterpret_cast<float *>(gbase + scring + slot * L::SCSLOT);
    const int nblk = (k.kbA + C < q.kblocks ? k.kbA + C : q.kblocks) - k.kbA;
    const int64_t bi0 = static_cast<int64_t>(k.tile) * kSmTileRows * q.kblocks + k.kbA;
    const int64_t gw = (bi0 >> 8) & ~int64_t{3};   // first constant of the TMA window
#pragma unroll
    for (int it = 2 * sw; it < 2 * sw + 2; ++it) {
      const int row = it * 32 + lane;
      const int rgi = row >> 5, wi = row & 31, gi = (wi & 15) >> 1, hi = 2 * (wi >> 4) + (wi & 1);
      const uint2 q8 = *reinterpret_cast<const uint2 *>(gbase + sq + row * 16 + (k.kbA & 15));
      const int64_t bi = bi0 + static_cast<int64_t>(row) * q.kblocks;
      float dA, dB;
      if (P.rawtma) {
        dA = s2w[(bi >> 8) - gw];
        dB = s2w[((bi + nblk - 1) >> 8) - gw];
      } else {
        const uint2 dw = *reinterpret_cast<const uint2 *>(gbase + sd + row * 8);
        dA = __uint_as_float(dw.x);
        dB = __uint_as_float(dw.y);
      }
      const int bnd = 256 - static_cast<int>(bi & 255);
      const float da = __fmul_rn(dA, kInvLambda), db = __fmul_rn(dB, kInvLambda);
#pragma unroll
      for (int i = 0; i < C; ++i) {
        const uint32_t b = ((i < 4 ? q8.x : q8.y) >> (8 * (i & 3))) & 0xFFu;
        scs[((i * 4 + rgi) * 8 + gi) * 4 + hi] = static_cast<float>(b) * (i < bnd ? da : db);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&sfull[slot]);
  };

  if (warp < kConsumerWarps) {
    // ======================= consumers =======================
    // Warp (rg, slice) owns tile rows 32 rg .. 32 rg + 31 (two 16-row MMA tiles)
    // and the chunk's blocks of parity `slice`.
    // ---- the level table: entry e (a code byte) at lut + 256 e + 4 lane holds
    // (bf16(lambda level[e >> 4]), bf16(lambda level[e & 15])) for every lane;
    // 16-byte stores of four lanes' copies at a time
    for (int i = threadIdx.x; i < 2048; i += kConsumerWarps * 32) {
      const int e = i >> 3, q4 = i & 7;
      const uint32_t v = static_cast<uint32_t>(P.lvl[e >> 4]) | (static_cast<uint32_t>(P.lvl[e & 15]) << 16);
      *reinterpret_cast<uint4 *>(gbase + lut + e * 256 + q4 * 16) = make_uint4(v, v, v, v);
    }
    named_barrier(kTableBar, kConsumerWarps * 32);

    const int rg = warp & 3, slice = warp >> 2;
    const uint32_t lreg = (lut & 0xFFFF0000u) | static_cast<uint32_t>(lane * 4);
    // code bytes of MMA row g (weight row 2g of a 16-row tile) and row g + 8
    // (weight row 2g + 1): row r of a 128-byte swizzled box holds 16-byte
    // chunk j at 16 (j ^ (r & 7)); this lane reads 8 bytes at byte 8c of a
    // block. Rows 2g + hh of the two tiles are 2048 bytes apart and share r & 7.
    const uint32_t hc = static_cast<uint32_t>(c >> 1);
    // this lane's K 16c .. 16c + 15 of a block are 16-byte chunks 2c and
    // 2c + 1 of its token's 128-byte row, swizzled by the row's low 3 bits (g)
    const uint32_t xo0 = static_cast<uint32_t>(((2 * c) ^ g) * 16), xo1 = static_cast<uint32_t>(((2 * c + 1) ^ g) * 16);
    uint32_t rbase[2], rxor[2];
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const uint32_t r = static_cast<uint32_t>(32 * rg + 2 * g + hh);
      rbase[hh] = r * 128u + static_cast<uint32_t>(8 * (c & 1));
      rxor[hh] = r & 7u;
    }
    float acc[2][NT][4];
#pragma unroll
    for (int t = 0; t < 2; ++t)
#pragma unroll
      for (int u = 0; u < NT; ++u) acc[t][u][0] = acc[t][u][1] = acc[t][u][2] = acc[t][u][3] = 0.f;

    Walk wk;
    walk_init(wk, ub, ue);
    Chunk cur;
    int chunk_idx = 0, seg_idx = 0;
    while (walk_next<C>(P, wk, cur)) {
      const int slot = chunk_idx % NS;
      // waits give the same answer on every lane: the MMAs below need the whole warp
      const uint32_t par = (chunk_idx / NS) & 1;
      if (!__all_sync(0xffffffffu, bar_wait(&full[slot], par, abort_flag, P.status) &&
                                       bar_wait(&sfull[slot], par, abort_flag, P.status)))
        break;
      const uint32_t cs = cring + slot * kCodeSlot;
      const uint32_t xs = xring + slot * L::XSLOT + g * 128;
      const uint32_t sc = scring + slot * L::SCSLOT + ((rg * 8 + g) * 4) * 4;
      const int f = cur.kb_s + (((cur.kb_s & 1) != slice) ? 1 : 0);
      const int nown = f < cur.kb_e ? (cur.kb_e - f + 1) / 2 : 0;
      // one 64-K block (chunk-local index kbl) of the warp's 32 rows
      auto block = [&](int kbl) {
        const uint32_t half = cs + static_cast<uint32_t>(kbl >> 2) * (kSmTileRows * 128u);
        const uint32_t jj = 2u * static_cast<uint32_t>(kbl & 3) + hc;
        uint2 w[2][2];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const uint32_t a = half + rbase[hh] + 16u * (jj ^ rxor[hh]);
          asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(w[0][hh].x), "=r"(w[0][hh].y) : "r"(a));
          asm volatile("ld.shared.v2.u32 {%0, %1}, [%2+2048];" : "=r"(w[1][hh].x), "=r"(w[1][hh].y) : "r"(a));
        }
        // activations: token 8u + g is row 8u + g of the block's swizzled box
        uint4 x[NT][2];
        const uint32_t xb = xs + static_cast<uint32_t>(kbl) * L::XBOX;
#pragma unroll
        for (int u = 0; u < NT; ++u) {
          x[u][0] = lds_u128(xb + u * 1024 + xo0);
          x[u][1] = lds_u128(xb + u * 1024 + xo1);
        }
        float4 sv;
        asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                     : "=f"(sv.x), "=f"(sv.y), "=f"(sv.z), "=f"(sv.w)
                     : "r"(sc + kbl * (kSmTileRows * 4)));
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
            const uint32_t a0 = lds_u32(prmt(wa, lreg, sel0));   // MMA row g,     K 4i, 4i+1 of the lane's 16
            const uint32_t a1 = lds_u32(prmt(wb, lreg, sel0));   // MMA row g + 8
            const uint32_t a2 = lds_u32(prmt(wa, lreg, sel1));   // MMA row g,     K 4i+2, 4i+3
            const uint32_t a3 = lds_u32(prmt(wb, lreg, sel1));   // MMA row g + 8
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
          const float s_lo = t == 0 ? sv.x : sv.z, s_hi = t == 0 ? sv.y : sv.w;
#pragma unroll
          for (int u = 0; u < NT; ++u) {
            acc[t][u][0] = fmaf(tmp[0][u][0] + tmp[1][u][0], s_lo, acc[t][u][0]);
            acc[t][u][1] = fmaf(tmp[0][u][1] + tmp[1][u][1], s_lo, acc[t][u][1]);
            acc[t][u][2] = fmaf(tmp[0][u][2] + tmp[1][u][2], s_hi, acc[t][u][2]);
            acc[t][u][3] = fmaf(tmp[0][u][3] + tmp[1][u][3], s_hi, acc[t][u][3]);
          }
        }
      };
      if (nown == D) {   // a whole chunk: no branches between the blocks
#pragma unroll
        for (int s = 0; s < D; ++s) block(f + 2 * s - cur.kbA);
      } else {
#pragma unroll
        for (int s = 0; s < D; ++s)
          if (s < nown) block(f + 2 * s - cur.kbA);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[slot]);

      if (cur.last) {   // hand the segment's sums to the epilogue warps
        const int eb = seg_idx & 1;
        if (!__all_sync(0xffffffffu, bar_wait(&eempty[eb], ((seg_idx >> 1) & 1) ^ 1, abort_flag, P.status))) break;
        const uint32_t ob = eb * L::EBUF + slice * kSmTileRows * L::EROW * 4;
#pragma unroll
        for (int t = 0; t < 2; ++t)
#pragma unroll
          for (int u = 0; u < NT; ++u) {
            const uint32_t row = 32 * rg + 16 * t + 2 * g;   // weight rows of MMA rows g and g + 8
            const uint32_t o = ob + (row * L::EROW + 8 * u + 2 * c) * 4;
            *reinterpret_cast<float2 *>(gbase + egap(o)) = make_float2(acc[t][u][0], acc[t][u][1]);
            *reinterpret_cast<float2 *>(gbase + egap(o + L::EROW * 4)) = make_float2(acc[t][u][2], acc[t][u][3]);
            acc[t][u][0] = acc[t][u][1] = acc[t][u][2] = acc[t][u][3] = 0.f;
          }
        __syncwarp();
        if (lane == 0) mbar_arrive(&efull[eb]);
        ++seg_idx;
      }
      ++chunk_idx;
    }
  } else if (warp == kProducerWarp) {
    // ======================= producer =======================
    // One thread: per chunk, wait for its slot (from the NS-th chunk on) and
    // request its copies.
    if (lane == 0) {
      Walk pwk;
      walk_init(pwk, ub, ue);
      Chunk k;
      int n = 0;   // chunks whose copies were requested
      while (walk_next<C>(P, pwk, k)) {
        const int slot = n % NS;
        if (n >= NS && !bar_wait(&empty[slot], ((n / NS) & 1) ^ 1, abort_flag, P.status, 32)) break;
        issue_tma(k, slot, n);
        ++n;
      }
      // do not leave while copies into this CTA's shared memory may be in flight
      if (*abort_flag) {
        for (int i = n - 1; i >= 0 && i >= n - NS; --i) {
          const uint64_t t0 = global_timer_ns();
          while (!mbar_try_wait(&full[i % NS], (i / NS) & 1) && global_timer_ns() - t0 < kWaitLimitNs) {
          }
        }
      }
    }
  } else if (warp < kScaleWarp0 + kScaleWarps) {
    // ======================= block scales =======================
    // The raw constants of chunk c are requested NS chunks ahead (when chunk
    // c - NS has been published, into the raw slot it used); per chunk: wait
    // for its slot, then for its raw constants, then publish its scales.
    Walk rwk, swk;
    walk_init(rwk, ub, ue);
    walk_init(swk, ub, ue);
    Chunk kr, k;
    int nraw = 0, n = 0;
    const bool issuer = sw == 0 && lane == 0;   // requests the raw constants of both warps
    if (P.rawtma) {
      if (issuer)
        for (; nraw < NS && walk_next<C>(P, rwk, kr); ++nraw) issue_raw_tma(kr, nraw);
      while (walk_next<C>(P, swk, k)) {
        const int slot = n % NS;
        if (n >= NS &&
            !__all_sync(0xffffffffu, bar_wait(&empty[slot], ((n / NS) & 1) ^ 1, abort_flag, P.status, 32)))
          break;
        if (!__all_sync(0xffffffffu, bar_wait(&rfull[slot], (n / NS) & 1, abort_flag, P.status))) break;
        publish_scales(k, slot);
        // the slot's raw constants were read by both warps: the second warp
        // arrives on sfull only after reading them
        bool ok = true;
        if (issuer && walk_next<C>(P, rwk, kr)) {
          ok = bar_wait(&sfull[slot], (n / NS) & 1, abort_flag, P.status);
          if (ok) {
            issue_raw_tma(kr, slot);
            ++nraw;
          }
        }
        if (!__all_sync(0xffffffffu, ok)) break;
        ++n;
      }
      // do not leave while copies into this CTA's shared memory may be in flight
      if (issuer && *abort_flag) {
        for (int i = nraw - 1; i >= 0 && i >= nraw - NS; --i) {
          const uint64_t t0 = global_timer_ns();
          while (!mbar_try_wait(&rfull[i % NS], (i / NS) & 1) && global_timer_ns() - t0 < kWaitLimitNs) {
          }
        }
      }
    } else {
    for (int i = 0; i < NS; ++i) {
      if (!walk_next<C>(P, rwk, kr)) break;
      issue_raw(kr, i);
      ++nraw;
    }
    while (walk_next<C>(P, swk, k)) {
      const int slot = n % NS;
      if (n >= NS &&
          !__all_sync(0xffffffffu, bar_wait(&empty[slot], ((n / NS) & 1) ^ 1, abort_flag, P.status, 32)))
        break;
      const int pend = nraw - n - 1;   // raw groups that may stay in flight
      if (pend >= 2)
        asm volatile("cp.async.wait_group 2;" ::: "memory");
      else if (pend == 1)
        asm volatile("cp.async.wait_group 1;" ::: "memory");
      else
        asm volatile("cp.async.wait_group 0;" ::: "memory");
      __syncwarp();
      publish_scales(k, slot);
      if (walk_next<C>(P, rwk, kr)) {
        issue_raw(kr, slot);
        ++nraw;
      }
      ++n;
    }
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    }
  } else {
    // ======================= epilogue =======================
    const int et = threadIdx.x - kEpiWarp0 * 32;   // 0..127: a tile row
    const int ew = et >> 5;
    if (P.pdl) grid_dep_wait();

    // ---- pieces of X A^T: 128 K each, every load issued before the MMAs ----
    // Inside each 64-K block the K order is permuted as in the weight path: lane
    // (g, c) holds K 16c .. 16c + 15 of a row, so its fragments are two 16-byte
    // loads per row and block. The piece that completes a linear's set adds all
    // of them in order and publishes sU = bf16(s X A^T).
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
      // the count releases the warp's partial sums (ordered before lane 0's add
      // by the warp barrier) and acquires the other pieces' for the last one
      unsigned long long old = 0;
      if (lane == 0) old = atom_add_acq_rel_gpu(&P.ucnt[p], 1ull);
      old = __shfl_sync(0xffffffffu, old, 0);
      __syncwarp();
      if (old + 1 == static_cast<unsigned long long>(q.uchunks)) {
        // the last piece: U = the pieces summed in piece order (16 loads in
        // flight per lane), sU = bf16(s U), then the linear's ready flag
        const int cols = 16 * r16 * MP / 4;   // float4 columns of one piece
        for (int col = lane; col < cols; col += 32) {
          const float4 *src4 = reinterpret_cast<const float4 *>(q.upart) + col;
          float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
          int cc = 0;
          for (; cc + 16 <= q.uchunks; cc += 16) {
            float4 v[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) v[e] = __ldcg(src4 + static_cast<int64_t>(cc + e) * cols);
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              a.x += v[e].x; a.y += v[e].y; a.z += v[e].z; a.w += v[e].w;
            }
          }
          for (; cc < q.uchunks; ++cc) {
            const float4 v = __ldcg(src4 + static_cast<int64_t>(cc) * cols);
            a.x += v.x; a.y += v.y; a.z += v.z; a.w += v.w;
          }
          const int j = (4 * col) / MP, t0 = (4 * col) % MP;
          const float uv[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
          for (int e = 0; e < 4; ++e)
            if (j < q.r && t0 + e < P.M)
              q.sU[static_cast<int64_t>(t0 + e) * q.r + j] = __bfloat16_as_ushort(__float2bfloat16_rn(q.s * uv[e]));
        }
        __syncwarp();   // the release below covers the whole warp's sU stores
        if (lane == 0) st_release_gpu_u64(&P.flags[G + p], P.epoch);
      }
    }

    // ---- finished segments ----
    // Before waiting for a segment that finishes a tile, the epilogue already
    // fetches that linear's sU (once per CTA and linear) and the tile's rows of
    // B, so only the sums and the stores remain after the wait.
    float *su_s = reinterpret_cast<float *>(gbase + sus);
    int su_p = -1;   // the linear whose sU su_s holds
    Walk wk;
    walk_init(wk, ub, ue);
    Chunk k;
    int seg_idx = 0;
    const int64_t self = blockIdx.x;
    while (walk_next<C>(P, wk, k)) {
      if (!k.last) continue;
      const SmProblem &q = P.p[k.p];
      const int64_t n = static_cast<int64_t>(k.tile) * kSmTileRows + et;
      const bool tile_first = k.seg_lo == 0, tile_last = k.seg_hi == q.kblocks;
      // rows of B held in registers across the wait: all 64 ranks for 8
      // tokens, the first 32 for 16 (the rest is loaded after it)
      constexpr int BPRE = NT == 2 ? 4 : 8;
      uint4 bpre[BPRE];
      const uint4 *brow = reinterpret_cast<const uint4 *>(q.B + n * q.r);
      if (tile_first) {
        if (k.p != su_p) {
          // the barrier also ends every read of su_s for the previous linear;
          // every path through a segment passes a barrier after reading epi_cmd[1]
          if (q.sU_in == nullptr && et == 0)
            epi_cmd[1] = wait_word(&P.flags[G + k.p], P.epoch, abort_flag, P.status) ? 1 : 0;
          named_barrier(kEpiBar, kEpiWarps * 32);
          if (q.sU_in == nullptr && epi_cmd[1] == 0) break;
          const uint16_t *sUp = q.sU_in ? q.sU_in : q.sU;
          for (int i = et; i < P.M * q.r; i += kEpiWarps * 32) {
            const int t = i / q.r, j = i % q.r;
            su_s[t * 64 + j] = __uint_as_float(static_cast<uint32_t>(__ldcg(sUp + i)) << 16);
          }
          su_p = k.p;
        }
        if (n < q.N) {
#pragma unroll
          for (int j8 = 0; j8 < BPRE; ++j8)
            if (j8 < q.r / 8) bpre[j8] = __ldg(brow + j8);
        }
      }
      const int eb = seg_idx & 1;
      // one thread waits and the barrier hands its answer to the others, so
      // all 128 leave together on a timeout (every later path passes a
      // barrier before epi_cmd[2] is written again)
      if (et == 0) epi_cmd[2] = bar_wait(&efull[eb], (seg_idx >> 1) & 1, abort_flag, P.status, 64) ? 1 : 0;
      named_barrier(kEpiBar, kEpiWarps * 32);
      if (epi_cmd[2] == 0) break;
      float sum[MP];
#pragma unroll
      for (int t = 0; t < MP; t += 4) {
        const uint32_t o = eb * L::EBUF + (et * L::EROW + t) * 4;
        const float4 a = *reinterpret_cast<const float4 *>(gbase + egap(o));
        const float4 b = *reinterpret_cast<const float4 *>(gbase + egap(o + kSmTileRows * L::EROW * 4));
        sum[t] = a.x + b.x;
        sum[t + 1] = a.y + b.y;
        sum[t + 2] = a.z + b.z;
        sum[t + 3] = a.w + b.w;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&eempty[eb]);
      ++seg_idx;

      if (!tile_first) {
        // a later contributor: publish the partial for the CTA holding the tile's first block
        float *slot = P.slots + self * (MP * kSmTileRows);
#pragma unroll
        for (int t = 0; t < MP; ++t)
          if (t < P.M) slot[t * kSmTileRows + et] = sum[t];
        // the barrier orders every thread's stores before thread 0's release,
        // which is cumulative: the flag publishes all of them at GPU scope
        named_barrier(kEpiBar, kEpiWarps * 32);
        if (et == 0) st_release_gpu_u64(&P.flags[self], P.epoch);
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
        // four contributors' partials are loaded before they are added (in CTA order)
        constexpr int CB = MP == 8 ? 4 : 2;
        int bb = static_cast<int>(self) + 1;
        for (; bb + CB - 1 <= b1; bb += CB) {
          float v[CB][MP];
#pragma unroll
          for (int i = 0; i < CB; ++i) {
            const float *slot = P.slots + static_cast<int64_t>(bb + i) * (MP * kSmTileRows);
#pragma unroll
            for (int t = 0; t < MP; ++t) v[i][t] = t < P.M ? __ldcg(slot + t * kSmTileRows + et) : 0.f;
          }
#pragma unroll
          for (int i = 0; i < CB; ++i)
#pragma unroll
            for (int t = 0; t < MP; ++t) sum[t] += v[i][t];
        }
        for (; bb <= b1; ++bb) {
          const float *slot = P.slots + static_cast<int64_t>(bb) * (MP * kSmTileRows);
#pragma unroll
          for (int t = 0; t < MP; ++t)
            if (t < P.M) sum[t] += __ldcg(slot + t * kSmTileRows + et);
        }
        named_barrier(kEpiBar, kEpiWarps * 32);
        if (et == 0)
          for (int bb = static_cast<int>(self) + 1; bb <= b1; ++bb) P.flags[bb] = 0;
      } else {
        named_barrier(kEpiBar, kEpiWarps * 32);   // su_s is complete
      }
      // finish the tile: the LoRA term in fp32, then Y in bf16
      if (n < q.N) {
        float y[MP];
#pragma unroll
        for (int t = 0; t < MP; ++t) y[t] = sum[t];
#pragma unroll
        for (int j8 = 0; j8 < 8; ++j8) {
          if (j8 < q.r / 8) {
            const uint4 bv = j8 < BPRE ? bpre[j8 < BPRE ? j8 : 0] : __ldg(brow + j8);
            const uint32_t bw[4] = {bv.x, bv.y, bv.z, bv.w};
            float bj[8];
#pragma unroll
            for (int h = 0; h < 8; ++h)
              bj[h] = __uint_as_float((h & 1) ? (bw[h >> 1] & 0xFFFF0000u) : (bw[h >> 1] << 16));
#pragma unroll
            for (int t = 0; t < MP; ++t) {   // sU[t][8 j8 .. 8 j8 + 7] in two 16-byte loads (same address for all threads)
              const float4 sa = *reinterpret_cast<const float4 *>(su_s + t * 64 + 8 * j8);
              const float4 sb = *reinterpret_cast<const float4 *>(su_s + t * 64 + 8 * j8 + 4);
              y[t] = fmaf(sa.x, bj[0], y[t]);
              y[t] = fmaf(sa.y, bj[1], y[t]);
              y[t] = fmaf(sa.z, bj[2], y[t]);
              y[t] = fmaf(sa.w, bj[3], y[t]);
              y[t] = fmaf(sb.x, bj[4], y[t]);
              y[t] = fmaf(sb.y, bj[5], y[t]);
              y[t] = fmaf(sb.z, bj[6], y[t]);
              y[t] = fmaf(sb.w, bj[7], y[t]);
            }
          }
        }
#pragma unroll
        for (int t = 0; t < MP; ++t)
          if (t < P.M) q.Y[static_cast<int64_t>(t) * q.N + n] = __bfloat16_as_ushort(__float2bfloat16_rn(y[t]));
      }
      if (q.sU_in == nullptr && et == 0) {
        if (atomicAdd(&P.ucons[k.p], 1ull) + 1 == static_cast<unsigned long long>(q.tiles)) {   // the last user
          atomicExch(&P.ucnt[k.p], 0ull);
          atomicExch(&P.ucons[k.p], 0ull);
          P.flags[G + k.p] = 0;
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

// bf16(lambda * level[i]): the fp32 product rounded to nearest even (the
// levels and lambda are finite and far from the bf16 range limits).
uint16_t lambda_level_bf16(int i) {
  static const float levels[16] = QLORA_NF4_LEVELS;
  const float v = kLambda * levels[i];
  uint32_t b;
  std::memcpy(&b, &v, 4);
  return static_cast<uint16_t>((b + 0x7FFFu + ((b >> 16) & 1u)) >> 16);
}

struct SmWsLayout {
  size_t flags, slots, total;
  size_t upart[kSmMaxProblems], su[kSmMaxProblems];
};

SmWsLayout sm_ws_layout(const SmallProblem *pr, int count, int64_t M) {
  SmWsLayout w{};
  const size_t G = static_cast<size_t>(device_sm_count());
  const int MP = M <= 8 ? 8 : 16;
  size_t off = 0;
  w.flags = off;   // [G] published partials, then [kSmMaxProblems] sU ready
  off += up256((G + kSmMaxProblems) * 8);
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
    SmHead &H = P.h;
    H.count = n;
    H.M = static_cast<int32_t>(M);
    for (int i = 0; i < 16; ++i) H.lvl[i] = lambda_level_bf16(i);
    const uint32_t mp = M > 8 ? 16 : 8;
    bool all3d = true;
    int64_t wu = 0;
    int32_t uu = 0;
    for (int i = 0; i < n; ++i) {
      if (!encode_2d(&P.tm_codes[i], CU_TENSOR_MAP_DATA_TYPE_UINT8, q[i].codes, static_cast<uint64_t>(q[i].K / 2),
                     static_cast<uint64_t>(q[i].N), static_cast<uint64_t>(q[i].K / 2), 128, kSmTileRows,
                     CU_TENSOR_MAP_SWIZZLE_128B))
        return cudaErrorInvalidValue;
      // activations as [K/64 blocks][M tokens][64]: one box holds a chunk's
      // 8 blocks for MP tokens, each token row 128 bytes, swizzled
      const uint64_t xd[3] = {64, static_cast<uint64_t>(M), static_cast<uint64_t>(q[i].K / kBlock)};
      const uint64_t xs[2] = {static_cast<uint64_t>(q[i].K) * 2, 128};
      const uint32_t xb[3] = {64, mp, static_cast<uint32_t>(kChunkBlocks)};
      all3d = all3d && encode_3d(&P.tm_x[i], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, q[i].X, xd, xs, xb,
                                 CU_TENSOR_MAP_SWIZZLE_128B);
      SmProblem &p = H.p[i];
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
    if (!all3d)   // else one 2-D box per block, for every linear of the launch
      for (int i = 0; i < n; ++i)
        if (!encode_2d(&P.tm_x[i], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, q[i].X, static_cast<uint64_t>(q[i].K),
                       static_cast<uint64_t>(M), static_cast<uint64_t>(q[i].K) * 2, 64, mp,
                       CU_TENSOR_MAP_SWIZZLE_128B))
          return cudaErrorInvalidValue;
    H.x3d = all3d ? 1 : 0;
    // raw constants by TMA when every linear allows it: q8 rows a multiple
    // of 16 bytes, a window of 256 second-level constants covering a chunk's
    // 128 rows (at most 480 blocks a row), 16-byte aligned arrays
    bool rawtma = true;
    for (int i = 0; i < n && rawtma; ++i) {
      const int64_t kb = q[i].K / kBlock;
      const uint64_t ngroups = static_cast<uint64_t>((q[i].N * kb + kGroup - 1) / kGroup);
      rawtma = kb % 16 == 0 && kb <= 480 && reinterpret_cast<uintptr_t>(q[i].scale8) % 16 == 0 &&
               reinterpret_cast<uintptr_t>(q[i].scale2) % 16 == 0 &&
               encode_2d(&P.tm_q8[i], CU_TENSOR_MAP_DATA_TYPE_UINT8, q[i].scale8, static_cast<uint64_t>(kb),
                         static_cast<uint64_t>(q[i].N), static_cast<uint64_t>(kb), 16, kSmTileRows,
                         CU_TENSOR_MAP_SWIZZLE_NONE) &&
               encode_2d(&P.tm_s2[i], CU_TENSOR_MAP_DATA_TYPE_FLOAT32, q[i].scale2, ngroups, 1,
                         (ngroups * 4 + 15) / 16 * 16, 256, 1, CU_TENSOR_MAP_SWIZZLE_NONE);
    }
    H.rawtma = rawtma ? 1 : 0;
    H.w_units = wu;
    H.u_units = uu;
    H.epoch = next_epoch();
    H.flags = reinterpret_cast<uint64_t *>(wsb + w.flags);
    H.ucnt = static_cast<unsigned long long *>(counters);
    H.ucons = H.ucnt + kSmMaxProblems;
    H.slots = reinterpret_cast<float *>(wsb + w.slots);
    H.status = status;
    H.pdl = pdl ? 1 : 0;

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
