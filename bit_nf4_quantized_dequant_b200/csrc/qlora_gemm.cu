// Fused NF4-dequant + bf16 tcgen05 GEMM for the QLoRA linear layer.
//
// "QLoRA and Fine-Tuning on One Consumer GPU", section "The idea in one line":
// the frozen base stays in 4 bits and each weight tile is dequantised to bf16
// only for the moment it is used in a matmul. "QLoRA, in depth", section "The
// mechanism in brief": y = W x + (alpha / r) B A x, and the backward needs the
// activation gradient dX = dY W' + (alpha / r) (dY B) A but never dW.
//
// Both products are run "swap-AB": the dequantised weight tile is the UMMA A
// operand (weight rows for FWD, weight columns for DX), the tokens are the UMMA
// N dimension (BT up to 256), so each dequantised weight feeds 2 * BT flops.
//
//   FWD: D[n, t] = sum_k W'[n, k] X[t, k]  + sum_j Bl[n, j] sU[t, j]  -> Y[t, n]
//        A tile K-major (W' rows are contiguous along k).
//   DX:  D[k, t] = sum_n W'[n, k] dY[t, n] + sum_j Al[j, k] sT[t, j] -> dX[t, k]
//        A tile MN-major (W' rows are contiguous along k, the M dimension).
// The LoRA term rides along as extra K-steps of r (padded to 16/32/64) at the
// end of each tile's accumulation, from a shared-memory slice that TMA loads
// once per tile.
//
// Three rings decouple the producers from the consumers: packed codes (TMA ->
// dequantisers, deep, so codes are waiting when a dequantiser gets to them),
// activations (TMA -> MMA) and dequantised bf16 tiles (dequantisers -> MMA).
// Three groups of four warps dequantise every third K-step each, one thread
// per 64-weight block: a group needs about three MMA K-steps' time for one
// tile, so with two groups the MMA waited for them (three groups: the DX
// launch of the 2048-token attention projection 69 -> 65 us, bit-identical).
//
// Two variants share this source. Single CTA: UMMA M = 128, one CTA per tile;
// a K-step of a 256-token tile needs 512 tensor cycles but the dequantisation
// of its 128 x 64 weights takes longer, so this variant is bound by the
// dequantisers. CTA pair (cta_group::2, a cluster of two): UMMA M = 256 across
// the pair and a 512-token tile, issued as two N = 256 MMAs per K-slice into
// two accumulators that fill each CTA's TMEM; each CTA dequantises its own 128
// weight rows and loads 256 of the tokens (128 for each MMA), so every
// dequantised weight feeds twice the flops of the single-CTA tile with the same
// shared memory per CTA. The even CTA issues the MMAs; the odd CTA's producers
// and dequantisers signal the even CTA's barriers, and the even CTA's MMA
// completions are multicast to both; the odd CTA's dequantised tiles reach
// the even CTA through one forwarding thread (a single cluster-scope release
// per K-step instead of one per dequantiser warp). The launcher takes the pair
// for large token counts (see use_pair); qlora_set_gemm_schedule can force
// either variant.
//
// Scheduling: persistent CTAs (or pairs) take whole tiles (tile = blockIdx + i * gridDim).
// With a workspace and token tiles of at most 64, stream-K instead: the
// (tile, k-step) units are split evenly over all SMs, and tiles cut between
// CTAs are finished through fp32 partials in the workspace (see GemmParams).
//
// Warp roles (640 threads, 96 registers each; stream-K: 512): 0 codes
// producer, 1 MMA issuer and TMEM owner, 2 activation producer, 3 LoRA-slice
// producer, 4-7 epilogue (TMEM lane quadrant = warp % 4; results leave through
// shared memory and TMA stores), 8-11, 12-15 (and 16-19) the dequantiser
// groups. Persistent CTAs walk the tile
// list; the single-CTA TMEM accumulator is double-buffered so the epilogue of
// one tile overlaps the main loop of the next (a pair's two accumulators take
// all 512 columns: its next tile's MMAs wait for the epilogue, while its
// producers and dequantisers run ahead).
#include <atomic>

#include "qlora_device.cuh"

namespace qlora {
namespace {

// Dequantiser groups of four warps: three for whole tiles; two for stream-K
// (short token tiles, where the third group's registers cost more than it
// adds), so the block is 640 or 512 threads.
__host__ __device__ constexpr int dq_groups(bool streamk) { return streamk ? 2 : 3; }
__host__ __device__ constexpr int kernel_threads(bool streamk) { return 256 + 128 * dq_groups(streamk); }
constexpr int kTileRows = 128;                                // weight rows per CTA
constexpr int kKStage = 64;                                   // K per step (one NF4 block)
constexpr uint32_t kATileBytes = kTileRows * kKStage * 2;     // 16 KiB
constexpr uint32_t kCodeTileBytes = kTileRows * kKStage / 2;  // 4 KiB
constexpr int kEpiTokens = 32;                                // tokens per TMA store box
constexpr uint32_t kOutStageBytes = kTileRows * kEpiTokens * 2;   // 8 KiB

struct GemmParams {
  const uint8_t *scale8;
  const float *scale2;
  int32_t *status;
  int64_t N, K, M;
  int mode;        // 0 FWD, 1 DX, 2 SwiGLU FWD (h), 3 SwiGLU BWD (dg, du); 2 and 3 run the FWD main loop
  int bt;          // token tile: UMMA N (single CTA), or 512 = two N = 256 MMAs (pair)
  int bt_cta;      // tokens whose activations this CTA loads (bt, or 256 for a pair)
  int sx, sa, sc;  // ring depths: activations, dequantised tiles, codes
  int r_pad;       // LoRA K extent in smem (16, 32 or 64)
  int row_tiles;   // tiles along the weight dimension (128 rows, or 256 for a pair)
  int tok_tiles;
  int nk;          // main-loop K steps per tile
  // Stream-K (single CTA only): CTA b of G takes units [b*U/G, (b+1)*U/G) of
  // the U = tiles * nk (tile, k-step) units. A tile split between CTAs is
  // finished by the CTA that holds its k = 0 unit (the lowest one); every
  // other CTA working on the tile has it as its first segment and publishes
  // that partial (fp32, part + j * 128 * bt, column-major [bt][128]) by
  // setting flags[j] = epoch, a value unique to the launch. The finishing CTA
  // adds the partials in CTA order and clears the flags for the next launch.
  int streamk;
  uint64_t epoch;
  float *part;
  uint64_t *flags;
};

__host__ __device__ inline uint32_t lora_a_bytes(int r_pad) { return kTileRows * r_pad * 2; }
__host__ __device__ inline uint32_t lora_b_bytes(int bt_cta, int r_pad) {
  return ((static_cast<uint32_t>(bt_cta) * r_pad * 2 + 1023u) / 1024u) * 1024u;
}

__device__ __forceinline__ uint32_t lora_layout(int r_pad) {
  return r_pad == 16 ? kLayoutSW32 : (r_pad == 32 ? kLayoutSW64 : kLayoutSW128);
}

struct Smem {
  uint8_t *x, *a, *lb, *la, *out, *c;
  uint32_t x_bytes;
  uint64_t *xf, *xe, *af, *ae, *cf, *ce, *lf, *le, *accf, *acce, *drain, *peer_full, *dhf;
  uint32_t *tmem_holder;
  int *abort_flag;
};

__device__ __forceinline__ Smem carve(uint8_t *base, const GemmParams &p) {
  Smem s;
  s.x_bytes = static_cast<uint32_t>(p.bt_cta) * 128u;
  uint8_t *ptr = base;
  s.x = ptr;   ptr += static_cast<size_t>(p.sx) * s.x_bytes;
  s.a = ptr;   ptr += static_cast<size_t>(p.sa) * kATileBytes;
  s.lb = ptr;  ptr += lora_b_bytes(p.bt_cta, p.r_pad);
  s.la = ptr;  ptr += lora_a_bytes(p.r_pad);
  s.out = ptr; ptr += 2 * kOutStageBytes;
  s.c = ptr;   ptr += static_cast<size_t>(p.sc) * kCodeTileBytes;
  uint64_t *b = reinterpret_cast<uint64_t *>(ptr);
  s.xf = b;           s.xe = s.xf + p.sx;
  s.af = s.xe + p.sx; s.ae = s.af + p.sa;
  s.cf = s.ae + p.sa; s.ce = s.cf + p.sc;
  s.lf = s.ce + p.sc; s.le = s.lf + 1;
  s.accf = s.le + 1;  s.acce = s.accf + 2;
  s.drain = s.acce + 2;
  s.peer_full = s.drain + 1;
  s.dhf = s.peer_full + 1;
  s.tmem_holder = reinterpret_cast<uint32_t *>(s.dhf + 2);
  s.abort_flag = reinterpret_cast<int *>(s.tmem_holder + 1);
  return s;
}

// Slot and phase of a ring position, advanced without division.
struct RingPos {
  int slot;
  uint32_t phase;
  __device__ __forceinline__ void advance(int by, int slots) {
    slot += by;
    while (slot >= slots) {
      slot -= slots;
      phase ^= 1u;
    }
  }
};

// The (tile, k-step) units a CTA (or CTA pair) processes, in order: starting at
// (first_tile, first_k), k runs to nk and then continues at k = 0 of tile +
// stride, for `total` units. Data-parallel: first_k = 0, stride = CTA count,
// whole tiles. Stream-K: stride = 1 over a contiguous range of units.
struct Walk {
  int first_tile, first_k, stride, total, row_tiles;
};

// A position in a Walk, advanced without division; rt / tt are the tile's
// indices along weights / tokens.
struct StepPos {
  int tile, k, rt, tt;
  __device__ __forceinline__ void set_tile(const Walk &w) {
    rt = tile % w.row_tiles;
    tt = tile / w.row_tiles;
  }
  __device__ __forceinline__ void init(const Walk &w) {
    tile = w.first_tile;
    k = w.first_k;
    set_tile(w);
  }
  __device__ __forceinline__ void advance(int by, int nk, const Walk &w) {
    k += by;
    if (k >= nk) {
      while (k >= nk) {
        k -= nk;
        tile += w.stride;
      }
      set_tile(w);
    }
  }
};

// On an abort, wait (bounded) until the copies this thread issued into a ring
// have landed, so that no TMA write outlives the CTA's shared memory.
__device__ __forceinline__ void drain_ring(uint64_t *full, int slots, uint32_t issued_mask,
                                           uint32_t parity_bits) {
  for (int s = 0; s < slots; ++s) {
    if (!(issued_mask & (1u << s))) continue;
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(&full[s], (parity_bits >> s) & 1u) && global_timer_ns() - t0 < kWaitLimitNs) {
    }
  }
}

// One instantiation per (pair, mode, stream-K) so that each launch carries only
// the code of its own epilogue: the instruction cache is shared by all roles.
template <bool kPair, int kMode, bool kStreamK>
__global__ void __launch_bounds__(kernel_threads(kStreamK), 1)
    fused_nf4_gemm_kernel(const __grid_constant__ CUtensorMap tm_act,
                          const __grid_constant__ CUtensorMap tm_codes,
                          const __grid_constant__ CUtensorMap tm_lora_w,
                          const __grid_constant__ CUtensorMap tm_lora_act,
                          const __grid_constant__ CUtensorMap tm_out,
                          const __grid_constant__ CUtensorMap tm_aux,   // dH (mode 3), else unused
                          const GemmParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const Smem sm = carve(base, p);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  constexpr bool dx = kMode == 1;
  constexpr bool swiglu = kMode >= 2;
  // CTA pair: rank 0 (even CTA) issues the MMAs; rank 1 is its peer.
  const uint32_t rank = kPair ? cluster_ctarank() : 0u;
  const bool leader = rank == 0;
  const int ntiles = p.row_tiles * p.tok_tiles;
  Walk walk;
  walk.row_tiles = p.row_tiles;
  const int64_t units = static_cast<int64_t>(ntiles) * p.nk;
  // first unit of CTA j under the stream-K split
  auto unit_begin = [&](int64_t j) -> int64_t { return units * j / gridDim.x; };
  if constexpr (!kPair && kStreamK) {
    const int64_t u0 = unit_begin(blockIdx.x), u1 = unit_begin(blockIdx.x + 1);
    walk.first_tile = static_cast<int>(u0 / p.nk);
    walk.first_k = static_cast<int>(u0 % p.nk);
    walk.stride = 1;
    walk.total = static_cast<int>(u1 - u0);
  } else {
    const int first = kPair ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
    const int stride = kPair ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);
    const int nlt = ntiles > first ? (ntiles - first + stride - 1) / stride : 0;
    walk.first_tile = first;
    walk.first_k = 0;
    walk.stride = stride;
    walk.total = nlt * p.nk;
  }
  const int total_steps = walk.total;
  const int rows_per_tile = kPair ? 2 * kTileRows : kTileRows;
  const int row_off = static_cast<int>(rank) * kTileRows;     // this CTA's weight rows inside the tile
  const int tok_off = static_cast<int>(rank) * p.bt_cta;      // this CTA's tokens inside the tile
  // single CTA: two accumulators of bt columns (at least 64 so a 32-column load
  // of buffer 1 stays inside); pair: one tile of 512 columns (two N = 256 halves)
  const uint32_t tmem_cols =
      kPair ? 512u : (static_cast<uint32_t>(2 * p.bt) < 64u ? 64u : static_cast<uint32_t>(2 * p.bt));
  // The pair's token order inside a tile: CTA rank q loads tokens [256 q, 256 q + 256)
  // of the tile; MMA half h reads rows [128 h, 128 h + 128) of both CTAs' stages, so
  // accumulator column c (half c / 256, n = c % 256) holds token
  // (n < 128 ? 0 : 256) + 128 (c / 256) + n % 128. A 32-column chunk is 32 consecutive tokens.
  auto chunk_token = [&](int tt, int col) -> int {
    if constexpr (kPair) {
      const int n = col & 255;
      return tt * p.bt + (n < 128 ? 0 : 256) + 128 * (col >> 8) + (n & 127);
    } else {
      return tt * p.bt + col;
    }
  };
  volatile int *abort_flag = sm.abort_flag;

  if (threadIdx.x == 0) {
    const uint32_t per_step = kPair ? 8u : 4u;   // epilogue warps that arrive, pair-wide
    // dequantised tile ready: this CTA's four dequantiser warps, plus (even CTA of
    // a pair) the one forwarded arrival for the odd CTA's half
    const uint32_t a_arrivals = kPair && leader ? 5u : 4u;
    for (int i = 0; i < p.sx; ++i) { mbar_init(&sm.xf[i], 1); mbar_init(&sm.xe[i], 1); }
    for (int i = 0; i < p.sa; ++i) { mbar_init(&sm.af[i], a_arrivals); mbar_init(&sm.ae[i], 1); }
    for (int i = 0; i < p.sc; ++i) { mbar_init(&sm.cf[i], 1); mbar_init(&sm.ce[i], 4); }
    mbar_init(sm.lf, 1);
    mbar_init(sm.le, 1);
    for (int i = 0; i < 2; ++i) { mbar_init(&sm.accf[i], 1); mbar_init(&sm.acce[i], per_step); }
    mbar_init(sm.drain, 1);
    mbar_init(sm.peer_full, 1);
    mbar_init(&sm.dhf[0], 1);
    mbar_init(&sm.dhf[1], 1);
    *sm.abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_act);
    tma_prefetch_desc(&tm_codes);
    tma_prefetch_desc(&tm_lora_w);
    tma_prefetch_desc(&tm_lora_act);
    tma_prefetch_desc(&tm_out);
    if constexpr (kMode == 3) tma_prefetch_desc(&tm_aux);
  }
  if (warp == 1) {
    if constexpr (kPair) {
      tmem_alloc_pair(sm.tmem_holder, tmem_cols);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(sm.tmem_holder, tmem_cols);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (kPair) cluster_sync_all();   // the peer's barriers exist before anyone signals them
  tc_fence_after();
  const uint32_t tmem_base = *sm.tmem_holder;
  const int kb_row = static_cast<int>(p.K / kBlock);   // NF4 blocks per weight row

  // An mbarrier of the even CTA (this CTA's own when not paired).
  auto leader_bar = [&](uint64_t *bar) -> uint32_t {
    return kPair ? mapa_shared(smem_u32(bar), 0u) : smem_u32(bar);
  };
  auto arrive_leader = [&](uint64_t *bar) {
    if constexpr (kPair) mbar_arrive_cluster(mapa_shared(smem_u32(bar), 0u));
    else mbar_arrive(bar);
  };
  auto load_for_leader = [&](void *dst, const CUtensorMap *map, uint64_t *bar, int32_t x, int32_t y) {
    if constexpr (kPair) tma_load_2d_pair(dst, map, leader_bar(bar), x, y);
    else tma_load_2d(dst, map, bar, x, y);
  };

  if (warp == 0) {
    // ---------------- codes producer (this CTA's weight rows only) ----------------
    if (elect_one()) {
      uint32_t mask = 0, par = 0;
      bool ok = true;
      RingPos c{0, 0};
      StepPos sp;
      sp.init(walk);
      for (int it = 0; it < total_steps; ++it, c.advance(1, p.sc), sp.advance(1, p.nk, walk)) {
        const int s = c.slot;
        const uint32_t ph = c.phase;
        if (!mbar_wait(&sm.ce[s], ph ^ 1u, abort_flag, p.status)) { ok = false; break; }
        mbar_arrive_expect_tx(&sm.cf[s], kCodeTileBytes);
        uint8_t *cp = sm.c + static_cast<size_t>(s) * kCodeTileBytes;
        const int r0 = sp.rt * rows_per_tile + row_off;
        if (!dx) tma_load_2d(cp, &tm_codes, &sm.cf[s], sp.k * (kKStage / 2), r0);
        else     tma_load_2d(cp, &tm_codes, &sm.cf[s], r0 / 2, sp.k * kKStage);
        mask |= 1u << s;
        par = (par & ~(1u << s)) | (ph << s);
      }
      if (!ok) drain_ring(sm.cf, p.sc, mask, par);
    }
  } else if (warp == 2) {
    // ---------------- activation producer (this CTA's tokens) ----------------
    if (elect_one()) {
      uint32_t mask = 0, par = 0;
      bool ok = true;
      RingPos x{0, 0};
      StepPos sp;
      sp.init(walk);
      for (int it = 0; it < total_steps; ++it, x.advance(1, p.sx), sp.advance(1, p.nk, walk)) {
        const int s = x.slot;
        const uint32_t ph = x.phase;
        if (!mbar_wait(&sm.xe[s], ph ^ 1u, abort_flag, p.status)) { ok = false; break; }
        if (leader) mbar_arrive_expect_tx(&sm.xf[s], kPair ? 2 * sm.x_bytes : sm.x_bytes);
        load_for_leader(sm.x + static_cast<size_t>(s) * sm.x_bytes, &tm_act, &sm.xf[s], sp.k * kKStage,
                        sp.tt * p.bt + tok_off);
        mask |= 1u << s;
        par = (par & ~(1u << s)) | (ph << s);
      }
      if (!ok && leader) drain_ring(sm.xf, p.sx, mask, par);
    }
  } else if (warp == 3) {
    // ---------------- LoRA-slice producer ----------------
    if (elect_one()) {
      bool issued = false;
      uint32_t last_ph = 0;
      const uint32_t bytes_cta = lora_a_bytes(p.r_pad) + static_cast<uint32_t>(p.bt_cta) * p.r_pad * 2u;
      StepPos seg;
      seg.init(walk);
      int n_lora = 0;
      for (int done = 0; done < total_steps;) {
        const int len = p.nk - seg.k < total_steps - done ? p.nk - seg.k : total_steps - done;
        if (seg.k + len == p.nk) {   // this segment ends its tile: it carries the LoRA K-steps
          const int r0 = seg.rt * rows_per_tile + row_off;
          const uint32_t ph = static_cast<uint32_t>(n_lora) & 1u;
          if (!mbar_wait(sm.le, ph ^ 1u, abort_flag, p.status)) break;
          if (leader) mbar_arrive_expect_tx(sm.lf, kPair ? 2 * bytes_cta : bytes_cta);
          load_for_leader(sm.lb, &tm_lora_act, sm.lf, 0, seg.tt * p.bt + tok_off);
          if (!dx) {
            load_for_leader(sm.la, &tm_lora_w, sm.lf, 0, r0);
          } else {
            load_for_leader(sm.la, &tm_lora_w, sm.lf, r0, 0);
            load_for_leader(sm.la + p.r_pad * 128, &tm_lora_w, sm.lf, r0 + 64, 0);
          }
          issued = true;
          last_ph = ph;
          ++n_lora;
        }
        done += len;
        seg.advance(len, p.nk, walk);
      }
      if (*abort_flag && issued && leader) drain_ring(sm.lf, 1, 1u, last_ph);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer (the even CTA of a pair) ----------------
    if (kPair && !leader && elect_one()) {
      // Odd CTA of a pair: its four dequantiser warps arrive on its own af[slot]
      // (CTA scope); this thread passes each completed tile on to the even CTA's
      // af[slot] with one cluster-scope release, which the dequantisers would
      // otherwise each pay on every K-step.
      RingPos ar{0, 0};
      for (int it = 0; it < total_steps; ++it, ar.advance(1, p.sa)) {
        if (!mbar_wait(&sm.af[ar.slot], ar.phase, abort_flag, p.status)) break;
        mbar_arrive_cluster(leader_bar(&sm.af[ar.slot]));
      }
    }
    if (leader && elect_one()) {
      const uint32_t idesc = idesc_bf16(static_cast<uint32_t>(rows_per_tile),
                                        static_cast<uint32_t>(kPair ? 256 : p.bt), dx, false);
      const uint32_t lsw = lora_layout(p.r_pad);
      const uint32_t lsbo = 16u * static_cast<uint32_t>(p.r_pad);   // 8 rows of 2 r_pad bytes
      const uint32_t la_addr = smem_u32(sm.la), lb_addr = smem_u32(sm.lb);
      auto mma = [&](uint32_t d, uint64_t ad, uint64_t bd, uint32_t acc) {
        if constexpr (kPair) umma_bf16_pair(d, ad, bd, idesc, acc);
        else umma_bf16(d, ad, bd, idesc, acc);
      };
      auto commit = [&](uint64_t *bar) {
        if constexpr (kPair) umma_commit_pair(bar);
        else umma_commit(bar);
      };
      // K-step j of a slot: +32 bytes along K (K-major A) or +2 K-groups of 8 rows (MN-major A)
      const uint64_t a_desc0 = dx ? smem_desc(smem_u32(sm.a), 8192u, 1024u, kLayoutSW128)
                                  : smem_desc(smem_u32(sm.a), 16u, 1024u, kLayoutSW128);
      const uint64_t b_desc0 = smem_desc(smem_u32(sm.x), 16u, 1024u, kLayoutSW128);
      const uint32_t a_step = dx ? 2048u / 16u : 32u / 16u;
      bool ok = true, issued_any = false;
      RingPos xr{0, 0}, ar{0, 0};
      StepPos seg;
      seg.init(walk);
      int n_lora = 0;
      for (int done = 0, si = 0; done < total_steps && ok; ++si) {
        const int kb = seg.k;
        const int len = p.nk - kb < total_steps - done ? p.nk - kb : total_steps - done;
        const int buf = kPair ? 0 : si & 1;
        const uint32_t acc_ph = kPair ? static_cast<uint32_t>(si) & 1u : static_cast<uint32_t>(si >> 1) & 1u;
        if (!mbar_wait(&sm.acce[buf], acc_ph ^ 1u, abort_flag, p.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * p.bt);
        for (int k = 0; k < len; ++k, xr.advance(1, p.sx), ar.advance(1, p.sa)) {
          const int xs = xr.slot, as = ar.slot;
          if (!mbar_wait(&sm.xf[xs], xr.phase, abort_flag, p.status) ||
              !mbar_wait(&sm.af[as], ar.phase, abort_flag, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          // descriptors = slot-0 descriptors + (byte offset >> 4) in the start-address field
          const uint64_t a0 = a_desc0 + static_cast<uint64_t>((static_cast<uint32_t>(as) * kATileBytes) >> 4);
          const uint64_t b0 = b_desc0 + static_cast<uint64_t>((static_cast<uint32_t>(xs) * sm.x_bytes) >> 4);
#pragma unroll
          for (int j = 0; j < kKStage / 16; ++j) {
            mma(d_tmem, a0 + static_cast<uint64_t>(a_step * j), b0 + static_cast<uint64_t>(2 * j), (k | j) != 0);
            if constexpr (kPair)   // tokens of the second half: stage rows 128..255 (+16 KiB)
              mma(d_tmem + 256u, a0 + static_cast<uint64_t>(a_step * j), b0 + static_cast<uint64_t>(1024 + 2 * j),
                  (k | j) != 0);
          }
          issued_any = true;
          commit(&sm.xe[xs]);
          commit(&sm.ae[as]);
        }
        if (!ok) break;
        if (kb + len == p.nk) {
          // LoRA K-steps: [.. | B] x [.. | sU] (FWD) or [.. ; A] x [.. | sT] (DX)
          if (!mbar_wait(sm.lf, static_cast<uint32_t>(n_lora) & 1u, abort_flag, p.status)) { ok = false; break; }
          tc_fence_after();
          for (int j = 0; j < p.r_pad / 16; ++j) {
            const uint64_t ad = dx ? smem_desc(la_addr + 2048u * j, 128u * p.r_pad, 1024u, kLayoutSW128)
                                   : smem_desc(la_addr + 32u * j, 16u, lsbo, lsw);
            const uint64_t bd = smem_desc(lb_addr + 32u * j, 16u, lsbo, lsw);
            mma(d_tmem, ad, bd, 1u);
            if constexpr (kPair)   // second half: sU / sT rows 128..255
              mma(d_tmem + 256u, ad, smem_desc(lb_addr + 256u * p.r_pad + 32u * j, 16u, lsbo, lsw), 1u);
          }
          commit(sm.le);
          ++n_lora;
        }
        commit(&sm.accf[buf]);
        done += len;
        seg.advance(len, p.nk, walk);
      }
      if (!ok && issued_any) {
        // drain: wait until every MMA issued so far has finished reading/writing
        commit(sm.drain);
        const uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait(sm.drain, 0) && global_timer_ns() - t0 < kWaitLimitNs) {
        }
      }
    }
  } else if (warp < 8) {
    // ---------------- epilogue: TMEM -> bf16 -> smem -> TMA store ----------------
    const int q = warp & 3;                 // TMEM lane quadrant of this warp
    const int et = threadIdx.x - 128;       // 0..127 = this CTA's weight row inside the tile
    const int box_t = p.bt < kEpiTokens ? p.bt : kEpiTokens;
    const int nchunks = p.bt / box_t;   // a pair's tile: 16 chunks over both halves
    uint32_t chunk_count = 0;
    uint32_t dh_count = 0;   // dH chunk loads so far (SwiGLU backward): buffer and phase
    StepPos seg;
    seg.init(walk);
    const int64_t part_elems = static_cast<int64_t>(kTileRows) * p.bt;
    for (int done = 0, si = 0; done < total_steps; ++si) {
      const int kb = seg.k;
      const int len = p.nk - kb < total_steps - done ? p.nk - kb : total_steps - done;
      const int rt = seg.rt, tt = seg.tt;
      const bool head = kStreamK && kb > 0;             // the end of a tile whose start another CTA computes
      const bool tail = kStreamK && kb + len < p.nk;    // the start of a tile that the next CTA completes
      const int buf = kPair ? 0 : si & 1;
      const uint32_t acc_ph = kPair ? static_cast<uint32_t>(si) & 1u : static_cast<uint32_t>(si >> 1) & 1u;
      if (!mbar_wait(&sm.accf[buf], acc_ph, abort_flag, p.status)) break;
      tc_fence_after();
      const uint32_t taddr =
          tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(buf * p.bt);
      if (head) {
        // Publish this partial accumulator for the CTA that finishes the tile:
        // fp32, column-major [bt][128], staged chunk by chunk through the
        // (otherwise idle: a head is a CTA's first segment) output buffer and
        // written with bulk copies.
        float *dst = p.part + static_cast<int64_t>(blockIdx.x) * part_elems;
        float *stagef = reinterpret_cast<float *>(sm.out);
        const uint32_t chunk_bytes = static_cast<uint32_t>(box_t) * kTileRows * 4u;
        for (int c = 0; c < nchunks; ++c) {
          uint32_t v[32];
          tmem_ld32(taddr + static_cast<uint32_t>(c * box_t), v);
          tmem_ld_wait();
          if (c == nchunks - 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) arrive_leader(&sm.acce[buf]);
          }
          if (et == 0) bulk_wait_group_read<0>();   // the previous chunk's copy has left the buffer
          named_barrier(1, 128);
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (j < box_t) stagef[j * kTileRows + et] = __uint_as_float(v[j]);
          fence_proxy_async_smem();
          named_barrier(1, 128);
          if (et == 0) {
            bulk_store(dst + static_cast<int64_t>(c * box_t) * kTileRows, stagef, chunk_bytes);
            bulk_commit_group();
          }
          __syncwarp();
        }
        if (et == 0) {
          bulk_wait_group<0>();        // the partial is in global memory
          fence_proxy_async_global();
          __threadfence();
          st_release_gpu_u64(p.flags + blockIdx.x, p.epoch);
        }
        __syncwarp();
      } else if (swiglu) {
        // SwiGLU tile: weight rows 0..63 are gate rows and 64..127 the up rows
        // of the same 64 output columns (the weight is [Wg; Wu] interleaved in
        // 64-row chunks), so TMEM lanes 0..63 hold g and lanes 64..127 hold u
        // for the tile's tokens. g and u are rounded to bf16 (the compute dtype
        // of the layer outputs) and exchanged between the two halves through
        // shared memory, 32 tokens at a time.
        const bool gate = q < 2;
        const int hr = et & 63;
        const uint32_t dh_bytes = static_cast<uint32_t>(box_t) * 64u * 2u;
        auto dh_buf = [&](uint32_t k) {
          return reinterpret_cast<uint16_t *>(sm.out + kOutStageBytes + (k & 1u) * (kOutStageBytes / 2));
        };
        if (kMode == 3 && et == 0) {   // dH for the first 32 tokens of the tile
          mbar_arrive_expect_tx(&sm.dhf[dh_count & 1u], dh_bytes);
          tma_load_2d(dh_buf(dh_count), &tm_aux, &sm.dhf[dh_count & 1u], rt * 64, tt * p.bt);
        }
        for (int c = 0; c < nchunks; ++c, ++chunk_count) {
          uint32_t v[32];
          tmem_ld32(taddr + static_cast<uint32_t>(c * box_t), v);
          tmem_ld_wait();
          if (c == nchunks - 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) arrive_leader(&sm.acce[buf]);
          }
          if constexpr (kMode == 2) {
            // h = bf16(silu(g) * u) -> H[tokens, 64 columns]
            uint8_t *cb = sm.out + (chunk_count & 1u) * kOutStageBytes;
            uint16_t *ux = reinterpret_cast<uint16_t *>(cb);          // [32 tokens][64] u
            uint16_t *hs = reinterpret_cast<uint16_t *>(cb + 4096);   // [32 tokens][64] h
            if (et == 0) bulk_wait_group_read<1>();   // the store that last used this buffer has read it
            named_barrier(1, 128);
            if (!gate) {
#pragma unroll
              for (int j = 0; j < 32; ++j)
                if (j < box_t) ux[j * 64 + hr] = __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(v[j])));
            }
            named_barrier(1, 128);
            if (gate) {
#pragma unroll
              for (int j = 0; j < 32; ++j) {
                if (j < box_t) {
                  const float g = __bfloat162float(__float2bfloat16_rn(__uint_as_float(v[j])));
                  const float u = __uint_as_float(static_cast<uint32_t>(ux[j * 64 + hr]) << 16);
                  const float h = __fdividef(g, 1.f + __expf(-g)) * u;
                  hs[j * 64 + hr] = __bfloat16_as_ushort(__float2bfloat16_rn(h));
                }
              }
            }
            fence_proxy_async_smem();
            named_barrier(1, 128);
            if (et == 0) {
              tma_store_2d(&tm_out, hs, rt * 64, tt * p.bt + c * box_t);
              bulk_commit_group();
            }
          } else {
            // dg = dh * u * silu'(g), du = dh * silu(g) -> dGU[tokens, 128 rows]
            uint16_t *xch = reinterpret_cast<uint16_t *>(sm.out);   // [32 tokens][128] g | u, then dg | du
            if (c + 1 < nchunks && et == 0) {   // dH of the next 32 tokens into the other buffer
              const uint32_t k = dh_count + 1;
              mbar_arrive_expect_tx(&sm.dhf[k & 1u], dh_bytes);
              tma_load_2d(dh_buf(k), &tm_aux, &sm.dhf[k & 1u], rt * 64, tt * p.bt + (c + 1) * box_t);
            }
            if (et == 0) bulk_wait_group_read<0>();   // the previous store has read the buffer
            named_barrier(1, 128);
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (j < box_t) xch[j * 128 + et] = __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(v[j])));
            mbar_wait(&sm.dhf[dh_count & 1u], (dh_count >> 1) & 1u, abort_flag, p.status);
            named_barrier(1, 128);
            const uint16_t *dhb = dh_buf(dh_count);
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              if (j < box_t) {
                const float own = __uint_as_float(static_cast<uint32_t>(xch[j * 128 + et]) << 16);
                const float other = __uint_as_float(static_cast<uint32_t>(xch[j * 128 + (et ^ 64)]) << 16);
                const float g = gate ? own : other, u = gate ? other : own;
                const float d = __uint_as_float(static_cast<uint32_t>(dhb[j * 64 + hr]) << 16);
                const float sg = __frcp_rn(1.f + __expf(-g));
                v[j] = __float_as_uint(gate ? d * u * sg * (1.f + g * (1.f - sg)) : d * g * sg);
              }
            }
            named_barrier(1, 128);   // every exchange read is done
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (j < box_t) xch[j * 128 + et] = __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(v[j])));
            fence_proxy_async_smem();
            named_barrier(1, 128);
            if (et == 0) {
              tma_store_2d(&tm_out, xch, rt * kTileRows, tt * p.bt + c * box_t);
              bulk_commit_group();
            }
            ++dh_count;
          }
          __syncwarp();
        }
      } else {
        // tail: CTAs blockIdx.x + 1 .. blockIdx.x + n_peers hold the rest of this tile
        int n_peers = 0, n_smem = 0;
        const float *peer = p.part + static_cast<int64_t>(blockIdx.x + 1) * part_elems;
        const float *peer_s = reinterpret_cast<const float *>(sm.x);
        if (tail) {
          const int64_t tile_end = static_cast<int64_t>(seg.tile + 1) * p.nk;
          while (static_cast<int64_t>(blockIdx.x) + n_peers + 1 < gridDim.x &&
                 unit_begin(blockIdx.x + n_peers + 1) < tile_end)
            ++n_peers;
          // This is the CTA's last segment: its rings are idle, so the peers'
          // partials are brought into them with bulk copies (as many as fit;
          // any others are read from global memory).
          const uint32_t part_bytes = static_cast<uint32_t>(part_elems) * 4u;
          const int cap = static_cast<int>(static_cast<uint32_t>(sm.out - sm.x) / part_bytes);
          n_smem = n_peers < cap ? n_peers : cap;
          if (et == 0) {
            const uint64_t t0 = global_timer_ns();
            for (int j = 1; j <= n_peers; ++j) {
              uint64_t *flag = p.flags + blockIdx.x + j;
              while (ld_acquire_gpu_u64(flag) != p.epoch) {
                if (global_timer_ns() - t0 > kWaitLimitNs) {
                  *abort_flag = 1;
                  set_status(p.status, 6 /* QLORA_ERR_TIMEOUT */);
                  break;
                }
                __nanosleep(256);
              }
              *flag = 0;   // consumed: the next launch (same epoch under graph replay) waits again
            }
            __threadfence();
            fence_proxy_async_global();
            if (n_smem > 0) {
              mbar_arrive_expect_tx(sm.peer_full, part_bytes * static_cast<uint32_t>(n_smem));
              for (int j = 0; j < n_smem; ++j)
                bulk_load(sm.x + static_cast<size_t>(j) * part_bytes, peer + static_cast<int64_t>(j) * part_elems,
                          part_bytes, sm.peer_full);
            }
          }
          __syncwarp();
          if (n_smem > 0) mbar_wait(sm.peer_full, 0, abort_flag, p.status);
          named_barrier(1, 128);
          __threadfence();
        }
        for (int c = 0; c < nchunks; ++c, ++chunk_count) {
          uint32_t v[32];
          tmem_ld32(taddr + static_cast<uint32_t>(c * box_t), v);
          tmem_ld_wait();
          if (c == nchunks - 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) arrive_leader(&sm.acce[buf]);
          }
          if (n_peers > 0) {
            const int64_t off = static_cast<int64_t>(c * box_t) * kTileRows + et;
            for (int pj = 0; pj < n_smem; ++pj) {
#pragma unroll
              for (int j = 0; j < 32; ++j)
                if (j < box_t)
                  v[j] = __float_as_uint(__uint_as_float(v[j]) + peer_s[pj * part_elems + off + j * kTileRows]);
            }
            for (int pj = n_smem; pj < n_peers; ++pj) {
              float w[32];
#pragma unroll
              for (int j = 0; j < 32; ++j) w[j] = j < box_t ? __ldcg(peer + pj * part_elems + off + j * kTileRows) : 0.f;
#pragma unroll
              for (int j = 0; j < 32; ++j) v[j] = __float_as_uint(__uint_as_float(v[j]) + w[j]);
            }
          }
          uint16_t *stage = reinterpret_cast<uint16_t *>(sm.out + (chunk_count & 1u) * kOutStageBytes);
          if (et == 0) bulk_wait_group_read<1>();   // the store that last used this buffer has read it
          named_barrier(1, 128);
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (j < box_t) stage[j * kTileRows + et] = __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(v[j])));
          fence_proxy_async_smem();
          named_barrier(1, 128);
          if (et == 0) {
            tma_store_2d(&tm_out, stage, rt * rows_per_tile + row_off, chunk_token(tt, c * box_t));
            bulk_commit_group();
          }
          __syncwarp();   // reconverge before the next warp-wide TMEM load
        }
      }
      done += len;
      seg.advance(len, p.nk, walk);
    }
    if (et == 0) bulk_wait_group<0>();
  } else {
    // ---------------- dequantisers: kDqGroups groups, each on every kDqGroups-th K-step ----------------
    constexpr int kDqGroups = dq_groups(kStreamK);
    const int g = (threadIdx.x - 256) >> 7;     // group 0 .. kDqGroups - 1
    const int i = (threadIdx.x - 256) & 127;    // block slot inside the step
    // FWD: slot = weight row n (0..127), one block per row per step.
    // DX:  slot = (column block kb in 0..1) * 64 + weight row n (0..63).
    const int n_loc = dx ? (i & 63) : i;
    const int kb_loc = dx ? (i >> 6) : 0;
    const uint32_t code_off =
        dx ? static_cast<uint32_t>(n_loc * 64 + kb_loc * 32) : static_cast<uint32_t>(n_loc * 32);
    const uint32_t out_row = dx ? static_cast<uint32_t>(kb_loc * 8192 + (n_loc >> 3) * 1024 + (n_loc & 7) * 128)
                                : static_cast<uint32_t>((n_loc >> 3) * 1024 + (n_loc & 7) * 128);
    const uint32_t sw = static_cast<uint32_t>(n_loc & 7);
    // scale of this thread's block at step position sp (q8 = 0 outside the matrix)
    auto scale_at = [&](const StepPos &sp, int it, uint32_t &q8, float &d) {
      q8 = 0;
      d = 0.f;
      if (it >= total_steps) return;
      int64_t n, kb;
      if (!dx) {
        n = static_cast<int64_t>(sp.rt) * rows_per_tile + row_off + n_loc;
        kb = sp.k;
      } else {
        n = static_cast<int64_t>(sp.k) * kKStage + n_loc;
        kb = (static_cast<int64_t>(sp.rt) * rows_per_tile + row_off) / kBlock + kb_loc;
      }
      if (n < p.N && kb < kb_row) {
        const int64_t b = n * kb_row + kb;
        q8 = __ldg(p.scale8 + b);
        d = __ldg(p.scale2 + (b >> 8));
      }
    };
    // Scale loads run three of this group's steps ahead; the loop
    // is unrolled by three so each prefetched value stays in its own register
    // until it is used.
    uint32_t qv[3];
    float dv[3];
    StepPos pf;                    // position of the next prefetch
    pf.init(walk);
    pf.advance(g, p.nk, walk);
#pragma unroll
    for (int u = 0; u < 3; ++u) {
      scale_at(pf, kDqGroups * u + g, qv[u], dv[u]);
      pf.advance(kDqGroups, p.nk, walk);
    }
    RingPos cr{g, 0}, ar{g, 0};    // rings of depth >= kDqGroups: step g sits in slot g of phase 0
    bool ok = true;
    for (int j0 = 0; ok; j0 += 3) {
#pragma unroll
      for (int u = 0; u < 3; ++u) {
        const int it = kDqGroups * (j0 + u) + g;
        if (it >= total_steps) { ok = false; break; }
        const int cs = cr.slot, as = ar.slot;
        if (!mbar_wait(&sm.cf[cs], cr.phase, abort_flag, p.status) ||
            !mbar_wait(&sm.ae[as], ar.phase ^ 1u, abort_flag, p.status)) {
          ok = false;
          break;
        }
        const uint8_t *c = sm.c + static_cast<size_t>(cs) * kCodeTileBytes + code_off;
        const uint4 c0 = *reinterpret_cast<const uint4 *>(c);
        const uint4 c1 = *reinterpret_cast<const uint4 *>(c + 16);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.ce[cs]);   // codes are in registers: release the slot
        const Nf4Table t = make_table(block_scale(qv[u], dv[u]));
        uint8_t *a = sm.a + static_cast<size_t>(as) * kATileBytes + out_row;
        const uint32_t w[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
        for (int h = 0; h < 8; ++h) {
          uint32_t o[4];
          expand8(t, w[h], o);
          *reinterpret_cast<uint4 *>(a + ((static_cast<uint32_t>(h) ^ sw) * 16u)) =
              make_uint4(o[0], o[1], o[2], o[3]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.af[as]);   // CTA scope; the odd CTA's tiles are forwarded
        scale_at(pf, it + 3 * kDqGroups, qv[u], dv[u]);
        pf.advance(kDqGroups, p.nk, walk);
        cr.advance(kDqGroups, p.sc);
        ar.advance(kDqGroups, p.sa);
      }
    }
  }

  // Every role above ran on one elected lane (or left its loop on its own); the
  // warp is reconverged before the CTA barrier (an aligned barrier) and before
  // the warp-wide TMEM deallocation.
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if constexpr (kPair) cluster_sync_all();   // the pair is done with each other's smem and TMEM
  if (warp == 1) {
    tc_fence_after();
    if constexpr (kPair) tmem_dealloc_pair(tmem_base, tmem_cols);
    else tmem_dealloc(tmem_base, tmem_cols);
  }
}

CUtensorMapSwizzle lora_swizzle(int r_pad) {
  return r_pad == 16 ? CU_TENSOR_MAP_SWIZZLE_32B
                     : (r_pad == 32 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B);
}

constexpr int kPairRings[3] = {3, 5, 4};   // activation, dequantised-tile, code stages

size_t smem_bytes(int bt_cta, int r_pad, int sx, int sa, int sc) {
  return 1024 /* alignment slack */ + static_cast<size_t>(sx) * bt_cta * 128u +
         static_cast<size_t>(sa) * kATileBytes + lora_b_bytes(bt_cta, r_pad) + lora_a_bytes(r_pad) +
         2 * kOutStageBytes + static_cast<size_t>(sc) * kCodeTileBytes +
         static_cast<size_t>(2 * (sx + sa + sc) + 10) * 8 + 16;
}

// Ring depths that fit the shared-memory budget, in order of preference: at
// least four activation stages (TMA latency), codes several steps ahead, three
// dequantised tiles ahead of the MMA. A pair's K-step is twice as long and its
// dequantised tiles cross the pair before the MMA can use them, so it keeps
// more of them in flight and fewer activation stages.
void pick_rings(int bt_cta, int r_pad, bool pair, int &sx, int &sa, int &sc) {
  const size_t budget = 227 * 1024;
  if (pair) {
    sx = kPairRings[0];
    sa = kPairRings[1];
    sc = kPairRings[2];
    if (smem_bytes(bt_cta, r_pad, sx, sa, sc) <= budget) return;
  }
  for (sx = 8; sx >= 4; --sx) {
    for (sc = 6; sc >= 4; sc -= 2) {
      sa = 3;
      if (smem_bytes(bt_cta, r_pad, sx, sa, sc) <= budget) return;
    }
  }
  const int fallback[][3] = {{3, 3, 4}, {2, 3, 4}, {2, 3, 3}};   // dequantised-tile and code rings >= 3 groups
  for (const auto &f : fallback) {
    sx = f[0];
    sa = f[1];
    sc = f[2];
    if (smem_bytes(bt_cta, r_pad, sx, sa, sc) <= budget) return;
  }
}

}  // namespace

// Host-side tensor-map encoder (driver entry point, resolved once).
bool encode_2d(CUtensorMap *map, CUtensorMapDataType dtype, const void *base, uint64_t inner,
               uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
               CUtensorMapSwizzle swizzle);

namespace {
int token_tile(int64_t M) {
  if (M <= 16) return 16;
  if (M <= 32) return 32;
  if (M <= 64) return 64;
  if (M <= 128) return 128;
  return 256;
}

constexpr int kPairTokens = 512;   // token tile of a CTA pair (two N = 256 MMAs)

// The CTA pair runs the linear forward and dX only. Each dequantised weight
// feeds a 512-token tile instead of 256, and each CTA reads half as many
// activation bytes per flop, so it spends less energy per flop: in short
// bursts of launches it is a few percent slower than single CTAs, but once
// the board sits at its power cap (long runs; on the 2048-token attention
// projection after a few hundred steps) it is faster (step 157 us against
// 163-167 us). The automatic schedule takes it when its tiles fill the SM
// pairs about as well as single-CTA tiles fill the SMs.
bool use_pair(const GemmArgs &a) {
  const int sched = gemm_schedule();
  if (a.mode > 1 || sched == 1) return false;
  if (sched == 2) return a.M > 0;
  if (a.M < 2 * kPairTokens) return false;
  const int64_t rows = a.mode == 1 ? a.K : a.N;
  const int64_t sms = device_sm_count();
  const int bt = token_tile(a.M);
  const int64_t t_single = ((rows + kTileRows - 1) / kTileRows) * ((a.M + bt - 1) / bt);
  const int64_t t_pair = ((rows + 2 * kTileRows - 1) / (2 * kTileRows)) * ((a.M + kPairTokens - 1) / kPairTokens);
  const double eff_single = static_cast<double>(t_single) / static_cast<double>(((t_single + sms - 1) / sms) * sms);
  const int64_t pairs = sms / 2;
  const double eff_pair = static_cast<double>(t_pair) / static_cast<double>(((t_pair + pairs - 1) / pairs) * pairs);
  return eff_pair >= 0.95 * eff_single;
}

std::atomic<int> g_schedule{0};
}  // namespace

void set_gemm_schedule(int schedule) { g_schedule.store(schedule, std::memory_order_relaxed); }
int gemm_schedule() { return g_schedule.load(std::memory_order_relaxed); }

size_t fused_gemm_ws_bytes(int64_t M) {
  const size_t sms = static_cast<size_t>(device_sm_count());
  const size_t flags = (sms * 8 + 255) / 256 * 256;
  return flags + sms * kTileRows * static_cast<size_t>(token_tile(M)) * 4;
}

cudaError_t launch_fused_gemm(const GemmArgs &a, cudaStream_t st) {
  GemmParams p{};
  p.scale8 = a.scale8;
  p.scale2 = a.scale2;
  p.status = a.dev_status;
  p.N = a.N;
  p.K = a.K;
  p.M = a.M;
  p.mode = a.mode;
  const int bt = token_tile(a.M);
  const bool pair = use_pair(a);
  p.bt = pair ? kPairTokens : bt;
  p.bt_cta = pair ? kPairTokens / 2 : bt;
  p.r_pad = a.r <= 16 ? 16 : (a.r <= 32 ? 32 : 64);
  pick_rings(p.bt_cta, p.r_pad, pair, p.sx, p.sa, p.sc);
  const int64_t rows = a.mode == 1 ? a.K : a.N;         // weight extent along UMMA M
  const int rows_per_tile = pair ? 2 * kTileRows : kTileRows;
  p.row_tiles = static_cast<int>((rows + rows_per_tile - 1) / rows_per_tile);
  p.tok_tiles = static_cast<int>((a.M + p.bt - 1) / p.bt);
  p.nk = static_cast<int>(a.mode != 1 ? a.K / kKStage : (a.N + kKStage - 1) / kKStage);

  CUtensorMap tm_act, tm_codes, tm_lw, tm_la, tm_out, tm_aux;
  const CUtensorMapSwizzle lsw = lora_swizzle(p.r_pad);
  const uint32_t box_t = bt < kEpiTokens ? bt : kEpiTokens;
  const uint32_t bt_cta = static_cast<uint32_t>(p.bt_cta);
  bool ok = true;
  if (a.mode != 1) {
    ok &= encode_2d(&tm_act, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.act, a.K, a.M, a.K * 2, 64, bt_cta,
                    CU_TENSOR_MAP_SWIZZLE_128B);
    ok &= encode_2d(&tm_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.codes, a.K / 2, a.N, a.K / 2, 32,
                    kTileRows, CU_TENSOR_MAP_SWIZZLE_NONE);
    ok &= encode_2d(&tm_lw, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.lora_w, a.r, a.N, a.r * 2, p.r_pad,
                    kTileRows, lsw);
    if (a.mode == 2)   // H [M, N / 2], 64 columns per tile
      ok &= encode_2d(&tm_out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.out, a.N / 2, a.M, a.N, 64, box_t,
                      CU_TENSOR_MAP_SWIZZLE_NONE);
    else
      ok &= encode_2d(&tm_out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.out, a.N, a.M, a.N * 2, kTileRows,
                      box_t, CU_TENSOR_MAP_SWIZZLE_NONE);
  } else {
    ok &= encode_2d(&tm_act, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.act, a.N, a.M, a.N * 2, 64, bt_cta,
                    CU_TENSOR_MAP_SWIZZLE_128B);
    ok &= encode_2d(&tm_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.codes, a.K / 2, a.N, a.K / 2, 64,
                    64, CU_TENSOR_MAP_SWIZZLE_NONE);
    ok &= encode_2d(&tm_lw, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.lora_w, a.K, a.r, a.K * 2, 64,
                    p.r_pad, CU_TENSOR_MAP_SWIZZLE_128B);
    ok &= encode_2d(&tm_out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.out, a.K, a.M, a.K * 2, kTileRows,
                    box_t, CU_TENSOR_MAP_SWIZZLE_NONE);
  }
  ok &= encode_2d(&tm_la, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.lora_act, a.r, a.M, a.r * 2, p.r_pad,
                  bt_cta, lsw);
  if (a.mode == 3)   // dH [M, N / 2]
    ok &= encode_2d(&tm_aux, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.aux, a.N / 2, a.M, a.N, 64, box_t,
                    CU_TENSOR_MAP_SWIZZLE_NONE);
  else
    tm_aux = tm_out;
  if (!ok) return cudaErrorInvalidValue;

  const size_t smem = smem_bytes(p.bt_cta, p.r_pad, p.sx, p.sa, p.sc);
  const int ntiles = p.row_tiles * p.tok_tiles;
  const int sms = device_sm_count();
  if (!pair) {
    int grid = ntiles < sms ? ntiles : sms;
    if (a.ws && bt <= 64 && a.mode <= 1) {
      // Stream-K over all SMs for short token tiles: a few weight-row tiles
      // would otherwise occupy a few SMs, and the fp32 partials that cross
      // CTAs are small. With 128- and 256-token tiles the partials (64 and
      // 128 KiB per split tile) cost more than the balance gains on B200.
      const int64_t units = static_cast<int64_t>(ntiles) * p.nk;
      grid = units < sms ? static_cast<int>(units) : sms;
      static std::atomic<uint64_t> launch_counter{0x51C0FFEE00000000ull};
      p.streamk = 1;
      p.epoch = ++launch_counter;
      const size_t flags = (static_cast<size_t>(sms) * 8 + 255) / 256 * 256;
      p.flags = static_cast<uint64_t *>(a.ws);
      p.part = reinterpret_cast<float *>(static_cast<uint8_t *>(a.ws) + flags);
    }
    auto go = [&](auto kernel) -> cudaError_t {
      cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
      if (e != cudaSuccess) return e;
      kernel<<<grid, kernel_threads(p.streamk != 0), smem, st>>>(tm_act, tm_codes, tm_lw, tm_la, tm_out, tm_aux, p);
      return cudaGetLastError();
    };
    switch (a.mode * 2 + p.streamk) {
      case 0: return go(fused_nf4_gemm_kernel<false, 0, false>);
      case 1: return go(fused_nf4_gemm_kernel<false, 0, true>);
      case 2: return go(fused_nf4_gemm_kernel<false, 1, false>);
      case 3: return go(fused_nf4_gemm_kernel<false, 1, true>);
      case 4: return go(fused_nf4_gemm_kernel<false, 2, false>);
      case 6: return go(fused_nf4_gemm_kernel<false, 3, false>);
      default: return cudaErrorInvalidValue;
    }
  }
  const void *pair_fn = a.mode == 0 ? reinterpret_cast<const void *>(fused_nf4_gemm_kernel<true, 0, false>)
                                    : reinterpret_cast<const void *>(fused_nf4_gemm_kernel<true, 1, false>);
  cudaError_t e = cudaFuncSetAttribute(pair_fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int pairs = ntiles < sms / 2 ? ntiles : sms / 2;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(2 * pairs));
  cfg.blockDim = dim3(kernel_threads(false));
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  void *args[] = {&tm_act, &tm_codes, &tm_lw, &tm_la, &tm_out, &tm_aux, &p};
  return cudaLaunchKernelExC(&cfg, pair_fn, args);
}

}  // namespace qlora
