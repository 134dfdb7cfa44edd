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
// * Codes go from global memory straight into registers (each consumer warp
//   keeps one chunk of its blocks in flight) and every code byte becomes a
//   bf16 pair with one PRMT and one shared-memory load: a 256-entry table of
//   (level[hi nibble], level[lo nibble]) pairs, one copy per lane in that
//   lane's own bank (64 KB), so the 32 lookups of a warp never conflict.
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
//   shared memory (padded rows: conflict-free 16-byte loads).
// * A producer warp stages the activations of each chunk of blocks with bulk
//   copies and precomputes the chunk's block scales into shared memory (one
//   16-byte load per block and lane for the consumers).
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
// QLORA_ERR_TIMEOUT in the status word and the CTA leaves. Counters in the
// workspace carry the launch's value in their high bits, so the workspace
// needs no initialisation; every counter and flag is cleared again by the
// launch that used it, so a captured launch can be replayed.
#include <atomic>
#include <chrono>

#include "qlora_device.cuh"

namespace qlora {
namespace {

constexpr int kSmMaxProblems = 16;
constexpr int kSmTileRows = 128;
constexpr int kConsumerWarps = 8;                    // 4 row groups x 2 K slices
constexpr int kProducerWarp = 8;
constexpr int kEpiWarp0 = 9;
constexpr int kEpiWarps = 4;
constexpr int kSmThreads = (kEpiWarp0 + kEpiWarps) * 32;   // 416
constexpr int kSmSlots = 3;                          // activation / scale ring depth
constexpr int kUnitK = 256;                          // K per piece of X A^T
constexpr uint32_t kLutBytes = 65536;                // 256 entries x 256 B (32 lanes x 4 B + unused half)
constexpr float kLambda = 1.43675f;
constexpr float kInvLambda = 1.0f / 1.43675f;
constexpr uint32_t kEpiBar = 1;                      // named barrier of the epilogue warps
constexpr uint64_t kCountBits = 20;

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
  SmProblem p[kSmMaxProblems];
  int32_t count, M;
  int64_t w_units;
  int32_t u_units;
  uint64_t epoch;          // launch value, 1 <= epoch < 2^44
  uint64_t *flags;         // [grid]: a contributor's partial is published
  float *slots;            // [grid][MP][128]: published partials
  uint64_t *sync;          // [count]: sU of a linear is ready
  uint64_t *ucnt;          // [count]: pieces of X A^T done
  uint64_t *ucons;         // [count]: tiles that have used sU
  int32_t *status;
  int32_t pdl;
};

// ---- small PTX helpers ------------------------------------------------------
__device__ __forceinline__ uint2 ldg_nc_v2(const void *p) {
  uint2 v;
  asm("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
  return v;
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
__device__ __forceinline__ float4 lds_f128(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr));
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

// Arrival on a counter word (launch value << 20 | count): a word that holds
// another launch's value (or anything left in fresh memory) counts as zero.
// Returns the count after this arrival.
__device__ __forceinline__ uint32_t epoch_arrive(uint64_t *ctr, uint64_t epoch) {
  unsigned long long *c = reinterpret_cast<unsigned long long *>(ctr);
  unsigned long long v = *reinterpret_cast<volatile unsigned long long *>(c);
  for (;;) {
    const unsigned long long base = (v >> kCountBits) == epoch ? v : (epoch << kCountBits);
    const unsigned long long got = atomicCAS(c, v, base + 1);
    if (got == v) return static_cast<uint32_t>((base + 1) & ((1ull << kCountBits) - 1));
    v = got;
  }
}

// Bounded wait until *w == v (GPU scope acquire); false on timeout.
__device__ __forceinline__ bool wait_word(const uint64_t *w, uint64_t v, volatile int *abort_flag, int32_t *status) {
  if (ld_acquire_gpu_u64(w) == v) return true;
  const uint64_t t0 = global_timer_ns();
  for (;;) {
    __nanosleep(256);
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
template <int MP>
struct Layout {
  static constexpr int C = 128 / MP;                        // blocks per chunk
  static constexpr uint32_t XROW = C * 128 + 16;            // bytes per token row of a chunk (padded)
  static constexpr uint32_t XSLOT = MP * XROW;
  static constexpr uint32_t XBYTES = kSmSlots * XSLOT;
  static constexpr uint32_t SCSLOT = C * kSmTileRows * 4;   // [block][row group][g][h] floats
  static constexpr uint32_t EROW = MP;                      // floats per row of an epilogue buffer
  static constexpr uint32_t EBUF = 2 * kSmTileRows * EROW * 4;   // [slice][row][token]
  static constexpr uint32_t SUBYTES = MP * 64 * 4;          // sU of one linear as float [t][64]
  static constexpr uint32_t BARBYTES = 128;
  static constexpr uint32_t REST = XBYTES + kSmSlots * SCSLOT + 2 * EBUF + SUBYTES + BARBYTES + 16;
  // dynamic shared memory to request: the table needs a 64 KB-aligned address
  // and the activation ring goes below it when there is room there
  static constexpr uint32_t request() {
    const uint32_t a = 2 * kLutBytes - 16 + REST - XBYTES;
    const uint32_t b = XBYTES + kLutBytes + REST;
    return (a > b ? a : b) + 16;
  }
};

template <int NT>
__global__ void __launch_bounds__(kSmThreads, 1) nf4_small_m_kernel(const __grid_constant__ SmParams P) {
  constexpr int MP = 8 * NT;
  using L = Layout<MP>;
  constexpr int C = L::C;
  constexpr int D = C / 2;   // own blocks of a consumer warp per chunk
  extern __shared__ __align__(1024) uint8_t smem[];

  if (P.pdl) grid_dep_launch();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;

  // ---- layout --------------------------------------------------------------
  const uint32_t base = smem_u32(smem);
  const uint32_t lut = (base + 0xFFFFu) & ~0xFFFFu;
  uint32_t xring, rest;
  if (lut - base >= L::XBYTES) {
    xring = base;
    rest = lut + kLutBytes;
  } else {
    xring = lut + kLutBytes;
    rest = xring + L::XBYTES;
  }
  const uint32_t scring = rest;
  const uint32_t ebuf = scring + kSmSlots * L::SCSLOT;
  const uint32_t sus = ebuf + 2 * L::EBUF;
  const uint32_t bars = sus + L::SUBYTES;
  const uint32_t end = bars + L::BARBYTES + 16;
  uint8_t *gbase = smem - base;   // generic pointer of shared address 0 (for plain C++ accesses)
  uint64_t *full = reinterpret_cast<uint64_t *>(gbase + bars);
  uint64_t *empty = full + kSmSlots;
  uint64_t *efull = empty + kSmSlots;
  uint64_t *eempty = efull + 2;
  volatile int *abort_flag = reinterpret_cast<volatile int *>(gbase + bars + L::BARBYTES);
  int *epi_cmd = reinterpret_cast<int *>(gbase + bars + L::BARBYTES + 4);

  if (end > base + dyn_smem_size()) {   // the host sized this; never expected
    if (threadIdx.x == 0) set_status(P.status, 7 /* QLORA_ERR_CUDA */);
    return;
  }

  // ---- init: the level table, zero activation rows beyond M, barriers ------
  {
    for (int i = threadIdx.x; i < 8192; i += kSmThreads) {
      const int e = i >> 5, ln = i & 31;
      const uint32_t lo = __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(kLambda, c_levels[e >> 4])));
      const uint32_t hi = __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(kLambda, c_levels[e & 15])));
      *reinterpret_cast<uint32_t *>(gbase + lut + e * 256 + ln * 4) = lo | (hi << 16);
    }
    for (int i = threadIdx.x; i < kSmSlots * (MP - P.M) * static_cast<int>(L::XROW / 16); i += kSmThreads) {
      const int per_slot = (MP - P.M) * static_cast<int>(L::XROW / 16);
      const int slot = i / per_slot, rem = i % per_slot;
      const int t = P.M + rem / static_cast<int>(L::XROW / 16), q = rem % static_cast<int>(L::XROW / 16);
      *reinterpret_cast<uint4 *>(gbase + xring + slot * L::XSLOT + t * L::XROW + q * 16) = make_uint4(0, 0, 0, 0);
    }
    if (threadIdx.x == 0) {
      for (int i = 0; i < kSmSlots; ++i) {
        mbar_init(&full[i], 32);
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
    const int rg = warp & 3, slice = warp >> 2;
    const uint32_t lreg = (lut & 0xFFFF0000u) | static_cast<uint32_t>(lane * 4);
    uint32_t ring[D][2][4];
    float acc[2][NT][4];
#pragma unroll
    for (int t = 0; t < 2; ++t)
#pragma unroll
      for (int u = 0; u < NT; ++u) acc[t][u][0] = acc[t][u][1] = acc[t][u][2] = acc[t][u][3] = 0.f;

    Walk wk;
    walk_init(wk, ub, ue);
    Chunk cur, nxt;
    bool have_cur = walk_next<C>(P, wk, cur);
    bool have_nxt = have_cur && walk_next<C>(P, wk, nxt);

    // row pointers of a chunk's tile for this lane: rows g, g + 8 of the two 16-row tiles
    auto own_first = [&](const Chunk &k) { return k.kb_s + (((k.kb_s & 1) != slice) ? 1 : 0); };
    auto own_count = [&](const Chunk &k) {
      const int f = own_first(k);
      return f < k.kb_e ? (k.kb_e - f + 1) / 2 : 0;
    };
    auto load_chunk_block = [&](uint32_t (&w)[2][4], const Chunk &k, int s) {
      const SmProblem &q = P.p[k.p];
      const int kb = own_first(k) + 2 * s;
      const int64_t half = q.K / 2;
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        const int64_t n = static_cast<int64_t>(k.tile) * kSmTileRows + 32 * rg + 16 * t + g;
        if (n < q.N) {
          const uint8_t *p0 = q.codes + n * half + static_cast<int64_t>(kb) * 32 + 8 * c;
          const uint2 a = ldg_nc_v2(p0), b = ldg_nc_v2(p0 + 8 * half);
          w[t][0] = a.x;
          w[t][1] = a.y;
          w[t][2] = b.x;
          w[t][3] = b.y;
        } else {
          w[t][0] = w[t][1] = w[t][2] = w[t][3] = 0x77777777u;   // code 7 = level 0
        }
      }
    };
    if (have_cur) {
      const int n0 = own_count(cur);
#pragma unroll
      for (int s = 0; s < D; ++s)
        if (s < n0) load_chunk_block(ring[s], cur, s);
    }

    int chunk_idx = 0, seg_idx = 0;
    while (have_cur) {
      const int slot = chunk_idx % kSmSlots;
      if (!mbar_wait(&full[slot], (chunk_idx / kSmSlots) & 1, abort_flag, P.status)) break;
      const uint32_t xs = xring + slot * L::XSLOT + g * L::XROW + 32 * c;
      const uint32_t sc = scring + slot * L::SCSLOT + ((rg * 8 + g) * 4) * 4;
      const int ncur = own_count(cur), nnxt = have_nxt ? own_count(nxt) : 0;
      const int f = own_first(cur);
#pragma unroll
      for (int s = 0; s < D; ++s) {
        if (s < ncur) {
          const int kbl = f + 2 * s - cur.kbA;
          uint4 x[NT][2];
#pragma unroll
          for (int u = 0; u < NT; ++u) {
            x[u][0] = lds_u128(xs + u * 8 * L::XROW + kbl * 128);
            x[u][1] = lds_u128(xs + u * 8 * L::XROW + kbl * 128 + 16);
          }
          const float4 sv = lds_f128(sc + kbl * (kSmTileRows * 4));
#pragma unroll
          for (int t = 0; t < 2; ++t) {
            float tmp[NT][4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const uint32_t wa = ring[s][t][i >> 1], wb = ring[s][t][2 + (i >> 1)];
              const uint32_t sel0 = 0x7604u | ((static_cast<uint32_t>(2 * i) & 3u) << 4);
              const uint32_t sel1 = 0x7604u | ((static_cast<uint32_t>(2 * i + 1) & 3u) << 4);
              const uint32_t a0 = lds_u32(prmt(wa, lreg, sel0));   // row g,     K 4i, 4i+1 of the lane's 16
              const uint32_t a1 = lds_u32(prmt(wb, lreg, sel0));   // row g + 8
              const uint32_t a2 = lds_u32(prmt(wa, lreg, sel1));   // row g,     K 4i+2, 4i+3
              const uint32_t a3 = lds_u32(prmt(wb, lreg, sel1));   // row g + 8
#pragma unroll
              for (int u = 0; u < NT; ++u) {
                const uint32_t b0 = (i == 0) ? x[u][0].x : (i == 1) ? x[u][0].z : (i == 2) ? x[u][1].x : x[u][1].z;
                const uint32_t b1 = (i == 0) ? x[u][0].y : (i == 1) ? x[u][0].w : (i == 2) ? x[u][1].y : x[u][1].w;
                if (i == 0)
                  mma_zero(tmp[u], a0, a1, a2, a3, b0, b1);
                else
                  mma_acc(tmp[u], a0, a1, a2, a3, b0, b1);
              }
            }
            const float s_lo = t == 0 ? sv.x : sv.z, s_hi = t == 0 ? sv.y : sv.w;
#pragma unroll
            for (int u = 0; u < NT; ++u) {
              acc[t][u][0] = fmaf(tmp[u][0], s_lo, acc[t][u][0]);
              acc[t][u][1] = fmaf(tmp[u][1], s_lo, acc[t][u][1]);
              acc[t][u][2] = fmaf(tmp[u][2], s_hi, acc[t][u][2]);
              acc[t][u][3] = fmaf(tmp[u][3], s_hi, acc[t][u][3]);
            }
          }
        }
        if (s < nnxt) load_chunk_block(ring[s], nxt, s);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[slot]);

      if (cur.last) {   // hand the segment's sums to the epilogue warps
        const int eb = seg_idx & 1;
        if (!mbar_wait(&eempty[eb], ((seg_idx >> 1) & 1) ^ 1, abort_flag, P.status)) break;
        float *dst = reinterpret_cast<float *>(gbase + ebuf + eb * L::EBUF) + slice * kSmTileRows * L::EROW;
#pragma unroll
        for (int t = 0; t < 2; ++t)
#pragma unroll
          for (int u = 0; u < NT; ++u) {
            const int row = 32 * rg + 16 * t + g;
            *reinterpret_cast<float2 *>(dst + row * L::EROW + 8 * u + 2 * c) = make_float2(acc[t][u][0], acc[t][u][1]);
            *reinterpret_cast<float2 *>(dst + (row + 8) * L::EROW + 8 * u + 2 * c) =
                make_float2(acc[t][u][2], acc[t][u][3]);
            acc[t][u][0] = acc[t][u][1] = acc[t][u][2] = acc[t][u][3] = 0.f;
          }
        __syncwarp();
        if (lane == 0) mbar_arrive(&efull[eb]);
        ++seg_idx;
      }
      cur = nxt;
      have_cur = have_nxt;
      if (have_cur) have_nxt = walk_next<C>(P, wk, nxt);
      ++chunk_idx;
    }
  } else if (warp == kProducerWarp) {
    // ======================= producer =======================
    Walk wk;
    walk_init(wk, ub, ue);
    Chunk k;
    int chunk_idx = 0;
    bool waited = false;
    constexpr int WPR = C / 4;              // 4-block words per row
    constexpr int RPI = 32 / WPR;           // rows per iteration
    while (walk_next<C>(P, wk, k)) {
      const int slot = chunk_idx % kSmSlots;
      if (!mbar_wait(&empty[slot], ((chunk_idx / kSmSlots) & 1) ^ 1, abort_flag, P.status)) break;
      const SmProblem &q = P.p[k.p];
      if (!waited) {
        if (P.pdl) grid_dep_wait();   // activations may come from the preceding launch
        waited = true;
      }
      const int nblk = (k.kbA + C < q.kblocks ? k.kbA + C : q.kblocks) - k.kbA;
      if (lane == 0) {
        const uint32_t bytes = static_cast<uint32_t>(nblk) * 128u;
        for (int t = 0; t < P.M; ++t)
          bulk_load(gbase + xring + slot * L::XSLOT + t * L::XROW,
                    q.X + static_cast<int64_t>(t) * q.K + static_cast<int64_t>(k.kbA) * 64, bytes, &full[slot]);
      }
      // block scales s = fp32(q8 * d) / lambda of the chunk's 128 rows
      float *scs = reinterpret_cast<float *>(gbase + scring + slot * L::SCSLOT);
      const bool fast = (q.kblocks & 3) == 0;
#pragma unroll 4
      for (int it = 0; it < kSmTileRows / RPI; ++it) {
        const int row = it * RPI + lane / WPR, wd = lane % WPR;
        const int64_t n = static_cast<int64_t>(k.tile) * kSmTileRows + row;
        const int kb0 = k.kbA + 4 * wd;
        float sv[4] = {0.f, 0.f, 0.f, 0.f};
        if (n < q.N && kb0 < k.kb_e && kb0 + 3 >= k.kb_s) {
          const int64_t bi = n * q.kblocks + kb0;
          if (fast) {
            const uint32_t q4 = __ldg(reinterpret_cast<const uint32_t *>(q.scale8 + bi));
            const float d = __ldg(q.scale2 + (bi >> 8));
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int kb = kb0 + i;
              if (kb >= k.kb_s && kb < k.kb_e)
                sv[i] = __fmul_rn(__fmul_rn(static_cast<float>((q4 >> (8 * i)) & 0xFFu), d), kInvLambda);
            }
          } else {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int kb = kb0 + i;
              if (kb >= k.kb_s && kb < k.kb_e) {
                const float d = __ldg(q.scale2 + ((bi + i) >> 8));
                sv[i] = __fmul_rn(__fmul_rn(static_cast<float>(__ldg(q.scale8 + bi + i)), d), kInvLambda);
              }
            }
          }
        }
        const int rgi = row >> 5, gi = row & 7, hi = (row >> 3) & 3;
#pragma unroll
        for (int i = 0; i < 4; ++i) scs[(((4 * wd + i) * 4 + rgi) * 8 + gi) * 4 + hi] = sv[i];
      }
      __syncwarp();
      if (lane == 0)
        mbar_arrive_expect_tx(&full[slot], static_cast<uint32_t>(P.M * nblk) * 128u);
      else
        mbar_arrive(&full[slot]);
      ++chunk_idx;
    }
    // do not leave while bulk copies into this CTA's shared memory may be in flight
    if (*abort_flag && chunk_idx > 0) {
      for (int i = chunk_idx - 1; i >= 0 && i >= chunk_idx - kSmSlots; --i) {
        const uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait(&full[i % kSmSlots], (i / kSmSlots) & 1) && global_timer_ns() - t0 < kWaitLimitNs) {
        }
      }
    }
  } else {
    // ======================= epilogue =======================
    const int et = threadIdx.x - kEpiWarp0 * 32;   // 0..127: a tile row
    const int ew = et >> 5;
    if (P.pdl) grid_dep_wait();

    // ---- pieces of X A^T ----
    for (int64_t qi = static_cast<int64_t>(blockIdx.x) * kEpiWarps + ew; qi < P.u_units;
         qi += static_cast<int64_t>(gridDim.x) * kEpiWarps) {
      int p = 0;
      for (int i = 1; i < P.count; ++i)
        if (qi >= P.p[i].u_unit0 && P.p[i].A) p = i;
      const SmProblem &q = P.p[p];
      const int ch = static_cast<int>(qi - q.u_unit0);
      const int k0 = ch * kUnitK, k1 = k0 + kUnitK < q.K ? k0 + kUnitK : q.K;
      const int r16 = (q.r + 15) / 16;
      float d[4][NT][4];
#pragma unroll
      for (int jt = 0; jt < 4; ++jt)
#pragma unroll
        for (int u = 0; u < NT; ++u) d[jt][u][0] = d[jt][u][1] = d[jt][u][2] = d[jt][u][3] = 0.f;
      for (int k = k0; k < k1; k += 16) {
        uint32_t b[NT][2];
#pragma unroll
        for (int u = 0; u < NT; ++u) {
          const int t = 8 * u + g;
          const uint32_t *xr = reinterpret_cast<const uint32_t *>(q.X + static_cast<int64_t>(t) * q.K + k + 2 * c);
          b[u][0] = t < P.M ? __ldg(xr) : 0u;
          b[u][1] = t < P.M ? __ldg(xr + 4) : 0u;
        }
#pragma unroll
        for (int jt = 0; jt < 4; ++jt) {
          if (jt < r16) {
            const int j0 = 16 * jt + g, j1 = j0 + 8;
            const uint32_t *a0p = reinterpret_cast<const uint32_t *>(q.A + static_cast<int64_t>(j0) * q.K + k + 2 * c);
            const uint32_t *a1p = reinterpret_cast<const uint32_t *>(q.A + static_cast<int64_t>(j1) * q.K + k + 2 * c);
            const uint32_t a0 = j0 < q.r ? __ldg(a0p) : 0u, a2 = j0 < q.r ? __ldg(a0p + 4) : 0u;
            const uint32_t a1 = j1 < q.r ? __ldg(a1p) : 0u, a3 = j1 < q.r ? __ldg(a1p + 4) : 0u;
#pragma unroll
            for (int u = 0; u < NT; ++u) mma_acc(d[jt][u], a0, a1, a2, a3, b[u][0], b[u][1]);
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
      __threadfence();
      __syncwarp();
      uint32_t n = 0;
      if (lane == 0) n = epoch_arrive(&P.ucnt[p], P.epoch);
      n = __shfl_sync(0xffffffffu, n, 0);
      if (n == static_cast<uint32_t>(q.uchunks)) {   // the last piece of this linear: sum in order
        __threadfence();
        for (int idx = lane; idx < P.M * q.r; idx += 32) {
          const int t = idx / q.r, j = idx % q.r;
          float acc_u = 0.f;
          for (int cc = 0; cc < q.uchunks; ++cc) acc_u += __ldcg(q.upart + (static_cast<int64_t>(cc) * (16 * r16) + j) * MP + t);
          q.sU[static_cast<int64_t>(t) * q.r + j] = __bfloat16_as_ushort(__float2bfloat16_rn(q.s * acc_u));
        }
        __threadfence();
        __syncwarp();
        if (lane == 0) {
          atomicExch(reinterpret_cast<unsigned long long *>(&P.ucnt[p]), 0ull);
          st_release_gpu_u64(&P.sync[p], P.epoch);
        }
      }
    }

    // ---- finished segments ----
    float *su_s = reinterpret_cast<float *>(gbase + sus);
    Walk wk;
    walk_init(wk, ub, ue);
    Chunk k;
    int seg_idx = 0;
    const int64_t self = blockIdx.x;
    while (walk_next<C>(P, wk, k)) {
      if (!k.last) continue;
      const int eb = seg_idx & 1;
      if (!mbar_wait(&efull[eb], (seg_idx >> 1) & 1, abort_flag, P.status)) break;
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
        __threadfence();
        named_barrier(kEpiBar, kEpiWarps * 32);
        if (et == 0) st_release_gpu_u64(&P.flags[self], P.epoch);
        continue;
      }
      if (!tile_last) {
        // owner of a split tile: add the later contributors' partials in CTA order
        const int64_t last_unit = q.w_unit0 + static_cast<int64_t>(k.tile + 1) * q.kblocks - 1;
        const int b1 = cta_of(last_unit, P.w_units, gridDim.x);
        bool ok = true;
        for (int bb = static_cast<int>(self) + 1; bb <= b1; ++bb) {
          if (et == 0) epi_cmd[0] = wait_word(&P.flags[bb], P.epoch, abort_flag, P.status) ? 1 : 0;
          named_barrier(kEpiBar, kEpiWarps * 32);
          ok = epi_cmd[0] != 0;
          named_barrier(kEpiBar, kEpiWarps * 32);
          if (!ok) break;
          const float *slot = P.slots + static_cast<int64_t>(bb) * (MP * kSmTileRows);
#pragma unroll
          for (int t = 0; t < MP; ++t)
            if (t < P.M) sum[t] += __ldcg(slot + t * kSmTileRows + et);
        }
        if (!ok) break;
        named_barrier(kEpiBar, kEpiWarps * 32);
        if (et == 0)
          for (int bb = static_cast<int>(self) + 1; bb <= b1; ++bb) P.flags[bb] = 0;
      }
      // finish the tile: the LoRA term in fp32, then Y in bf16
      if (q.sU_in == nullptr) {
        if (et == 0) epi_cmd[0] = wait_word(&P.sync[k.p], P.epoch, abort_flag, P.status) ? 1 : 0;
        named_barrier(kEpiBar, kEpiWarps * 32);
        if (epi_cmd[0] == 0) break;
      }
      const uint16_t *sUp = q.sU_in ? q.sU_in : q.sU;
      for (int i = et; i < P.M * q.r; i += kEpiWarps * 32) {
        const int t = i / q.r, j = i % q.r;
        const uint16_t v = q.sU_in ? __ldg(sUp + i) : __ldcg(sUp + i);
        su_s[t * 64 + j] = __uint_as_float(static_cast<uint32_t>(v) << 16);
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
        if (epoch_arrive(&P.ucons[k.p], P.epoch) == static_cast<uint32_t>(q.tiles)) {
          P.sync[k.p] = 0;
          atomicExch(reinterpret_cast<unsigned long long *>(&P.ucons[k.p]), 0ull);
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
  size_t flags, sync, slots, per_problem, total;
  size_t upart[kSmMaxProblems], su[kSmMaxProblems];
};

SmWsLayout sm_ws_layout(const SmallProblem *pr, int count, int64_t M) {
  SmWsLayout w{};
  const size_t G = static_cast<size_t>(device_sm_count());
  const int MP = M <= 8 ? 8 : 16;
  size_t off = 0;
  w.flags = off;
  off += up256(G * 8);
  w.sync = off;
  off += up256(3 * static_cast<size_t>(count) * 8);
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

cudaError_t launch_small_m(const SmallProblem *pr, int count, int64_t M, void *ws, bool pdl, int32_t *status,
                           cudaStream_t st) {
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
    P.sync = reinterpret_cast<uint64_t *>(wsb + w.sync);
    P.ucnt = P.sync + n;
    P.ucons = P.sync + 2 * n;
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
