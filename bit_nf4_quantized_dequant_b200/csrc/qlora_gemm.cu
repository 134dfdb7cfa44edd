// Fused NF4-dequant + bf16 tcgen05 GEMM for the QLoRA linear layer.
//
// "QLoRA and Fine-Tuning on One Consumer GPU", section "The idea in one line":
// the frozen base stays in 4 bits and each weight tile is dequantised to bf16
// only for the moment it is used in a matmul. "QLoRA, in depth", section "The
// mechanism in brief": y = W x + (alpha / r) B A x, and the backward needs the
// activation gradient dX = dY W' + (alpha / r) (dY B) A but never dW.
//
// Both products are run "swap-AB": the dequantised weight tile is the UMMA A
// operand (M = 128 weight rows or columns), the tokens are the UMMA N dimension
// (BT up to 256), so each dequantised tile feeds 2 * 128 * BT flops.
//
//   FWD: D[n, t] = sum_k W'[n, k] X[t, k]  + sum_j Bl[n, j] sU[t, j]  -> Y[t, n]
//        A tile K-major (W' rows are contiguous along k).
//   DX:  D[k, t] = sum_n W'[n, k] dY[t, n] + sum_j Al[j, k] sT[t, j] -> dX[t, k]
//        A tile MN-major (W' rows are contiguous along k, the M dimension).
// The LoRA term rides along as one extra K-step of r (padded to 16/32/64) whose
// operands TMA loads straight into a pipeline stage.
//
// Warp roles (512 threads): warp 0 TMA producer, warp 1 MMA issuer and TMEM
// owner, warps 4-7 epilogue (TMEM lane quadrant = warp % 4), warps 8-15
// dequantise (two threads per 64-weight block). Persistent CTAs walk the tile
// list; the TMEM accumulator is double-buffered so the epilogue of one tile
// overlaps the main loop of the next.
#include <cstdio>

#include "qlora_device.cuh"

namespace qlora {
namespace {

constexpr int kThreads = 512;
constexpr int kTileRows = 128;                 // UMMA M
constexpr int kKStage = 64;                    // K per pipeline stage (one NF4 block)
constexpr uint32_t kATileBytes = kTileRows * kKStage * 2;   // 16 KiB
constexpr uint32_t kCodeTileBytes = kTileRows * kKStage / 2;  // 4 KiB

struct GemmParams {
  const uint8_t *scale8;
  const float *scale2;
  uint16_t *out;
  int32_t *status;
  int64_t N, K, M;
  int mode;           // 0 FWD, 1 DX
  int bt;             // token tile (UMMA N)
  int stages;
  int r_pad;          // LoRA K extent in smem (16, 32 or 64)
  int row_tiles;      // tiles along the UMMA M dimension
  int tok_tiles;
  int nk;             // main-loop K steps per tile
};

__device__ __forceinline__ uint32_t lora_layout(int r_pad) {
  return r_pad == 16 ? kLayoutSW32 : (r_pad == 32 ? kLayoutSW64 : kLayoutSW128);
}

struct Smem {
  uint8_t *a, *b, *c;
  uint32_t b_stage_bytes;
  uint64_t *full, *afull, *empty, *accfull, *accempty, *drain;
  uint32_t *tmem_holder;
  int *abort_flag;
};

__device__ __forceinline__ Smem carve(uint8_t *base, const GemmParams &p) {
  Smem s;
  s.b_stage_bytes = static_cast<uint32_t>(p.bt) * 128u;
  s.a = base;
  s.b = s.a + static_cast<size_t>(p.stages) * kATileBytes;
  s.c = s.b + static_cast<size_t>(p.stages) * s.b_stage_bytes;
  uint64_t *bars = reinterpret_cast<uint64_t *>(s.c + static_cast<size_t>(p.stages) * kCodeTileBytes);
  s.full = bars;
  s.afull = bars + p.stages;
  s.empty = bars + 2 * p.stages;
  s.accfull = bars + 3 * p.stages;
  s.accempty = s.accfull + 2;
  s.drain = s.accempty + 2;
  s.tmem_holder = reinterpret_cast<uint32_t *>(s.drain + 1);
  s.abort_flag = reinterpret_cast<int *>(s.tmem_holder + 1);
  return s;
}

__global__ void __launch_bounds__(kThreads, 1)
    fused_nf4_gemm_kernel(const __grid_constant__ CUtensorMap tm_act,
                          const __grid_constant__ CUtensorMap tm_codes,
                          const __grid_constant__ CUtensorMap tm_lora_w,
                          const __grid_constant__ CUtensorMap tm_lora_act, const GemmParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const Smem sm = carve(base, p);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const bool dx = p.mode == 1;
  const int ntiles = p.row_tiles * p.tok_tiles;
  // two accumulators of bt columns; at least 64 so a 32-column load of buffer 1 stays inside
  const uint32_t tmem_cols = static_cast<uint32_t>(2 * p.bt) < 64u ? 64u : static_cast<uint32_t>(2 * p.bt);
  volatile int *abort_flag = sm.abort_flag;

  if (threadIdx.x == 0) {
    for (int i = 0; i < p.stages; ++i) {
      mbar_init(&sm.full[i], 1);
      mbar_init(&sm.afull[i], 8);   // one arrival per dequant warp
      mbar_init(&sm.empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.accfull[i], 1);
      mbar_init(&sm.accempty[i], 4);  // one arrival per epilogue warp
    }
    mbar_init(sm.drain, 1);
    *sm.abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_act);
    tma_prefetch_desc(&tm_codes);
    tma_prefetch_desc(&tm_lora_w);
    tma_prefetch_desc(&tm_lora_act);
  }
  if (warp == 1) {
    tmem_alloc(sm.tmem_holder, tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *sm.tmem_holder;

  const int kb_row = static_cast<int>(p.K / kBlock);   // NF4 blocks per weight row
  const int iters = p.nk + 1;                          // main K steps + the LoRA step

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (elect_one()) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_parity = 0, issued_mask = 0;
      const uint32_t act_bytes = static_cast<uint32_t>(p.bt) * 128u;
      const uint32_t lora_act_bytes = static_cast<uint32_t>(p.bt) * static_cast<uint32_t>(p.r_pad) * 2u;
      const uint32_t lora_w_bytes = static_cast<uint32_t>(kTileRows) * static_cast<uint32_t>(p.r_pad) * 2u;
      bool ok = true;
      for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
        const int rt = tile % p.row_tiles;
        const int tt = tile / p.row_tiles;
        const int r0 = rt * kTileRows;
        const int t0 = tt * p.bt;
        for (int k = 0; k < iters; ++k) {
          if (!mbar_wait(&sm.empty[stage], phase ^ 1, abort_flag, p.status)) { ok = false; break; }
          uint8_t *a = sm.a + static_cast<size_t>(stage) * kATileBytes;
          uint8_t *b = sm.b + static_cast<size_t>(stage) * sm.b_stage_bytes;
          uint8_t *c = sm.c + static_cast<size_t>(stage) * kCodeTileBytes;
          if (k < p.nk) {
            mbar_arrive_expect_tx(&sm.full[stage], act_bytes + kCodeTileBytes);
            tma_load_2d(b, &tm_act, &sm.full[stage], k * kKStage, t0);
            if (!dx) tma_load_2d(c, &tm_codes, &sm.full[stage], k * (kKStage / 2), r0);
            else     tma_load_2d(c, &tm_codes, &sm.full[stage], rt * (kTileRows / 2), k * kKStage);
          } else {
            mbar_arrive_expect_tx(&sm.full[stage], lora_act_bytes + lora_w_bytes);
            tma_load_2d(b, &tm_lora_act, &sm.full[stage], 0, t0);
            if (!dx) {
              tma_load_2d(a, &tm_lora_w, &sm.full[stage], 0, r0);
            } else {
              tma_load_2d(a, &tm_lora_w, &sm.full[stage], r0, 0);
              tma_load_2d(a + p.r_pad * 128, &tm_lora_w, &sm.full[stage], r0 + 64, 0);
            }
          }
          issued_mask |= 1u << stage;
          issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == p.stages) { stage = 0; phase ^= 1; }
        }
      }
      if (!ok) {
        // let copies already in flight land before the CTA's shared memory goes away
        for (int s = 0; s < p.stages; ++s) {
          if (!(issued_mask & (1u << s))) continue;
          const uint64_t t0 = global_timer_ns();
          while (!mbar_try_wait(&sm.full[s], (issued_parity >> s) & 1u) &&
                 global_timer_ns() - t0 < kWaitLimitNs) {
          }
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (elect_one()) {
      const uint32_t idesc = idesc_bf16(kTileRows, static_cast<uint32_t>(p.bt), dx, false);
      const uint32_t lora_sw = lora_layout(p.r_pad);
      const uint32_t lora_sbo = 16u * static_cast<uint32_t>(p.r_pad);   // 8 rows of 2 r_pad bytes
      int stage = 0;
      uint32_t phase = 0;
      int lt = 0;
      bool ok = true;
      bool issued_any = false;
      for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x, ++lt) {
        const int buf = lt & 1;
        const uint32_t acc_phase = (lt >> 1) & 1;
        if (!mbar_wait(&sm.accempty[buf], acc_phase ^ 1, abort_flag, p.status)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * p.bt);
        for (int k = 0; k < iters; ++k) {
          if (!mbar_wait(&sm.full[stage], phase, abort_flag, p.status) ||
              !mbar_wait(&sm.afull[stage], phase, abort_flag, p.status)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sm.a + static_cast<size_t>(stage) * kATileBytes);
          const uint32_t b_addr = smem_u32(sm.b + static_cast<size_t>(stage) * sm.b_stage_bytes);
          if (k < p.nk) {
#pragma unroll
            for (int j = 0; j < kKStage / 16; ++j) {
              const uint64_t ad = dx ? smem_desc(a_addr + 2048u * j, 8192u, 1024u, kLayoutSW128)
                                     : smem_desc(a_addr + 32u * j, 16u, 1024u, kLayoutSW128);
              const uint64_t bd = smem_desc(b_addr + 32u * j, 16u, 1024u, kLayoutSW128);
              umma_bf16(d_tmem, ad, bd, idesc, (k | j) != 0);
            }
          } else {
            for (int j = 0; j < p.r_pad / 16; ++j) {
              const uint64_t ad =
                  dx ? smem_desc(a_addr + 2048u * j, 128u * p.r_pad, 1024u, kLayoutSW128)
                     : smem_desc(a_addr + 32u * j, 16u, lora_sbo, lora_sw);
              const uint64_t bd = smem_desc(b_addr + 32u * j, 16u, lora_sbo, lora_sw);
              umma_bf16(d_tmem, ad, bd, idesc, 1u);
            }
          }
          issued_any = true;
          umma_commit(&sm.empty[stage]);
          if (++stage == p.stages) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        umma_commit(&sm.accfull[buf]);
      }
      if (!ok && issued_any) {
        // drain: wait until every MMA issued so far has finished reading/writing
        umma_commit(sm.drain);
        const uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait(sm.drain, 0) && global_timer_ns() - t0 < kWaitLimitNs) {
        }
      }
    }
  } else if (warp >= 4 && warp < 8) {
    // ---------------- epilogue ----------------
    const int q = warp & 3;                 // TMEM lane quadrant of this warp
    const int64_t ld = dx ? p.K : p.N;      // row length of the output
    const int64_t rows_total = dx ? p.K : p.N;
    int lt = 0;
    for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++lt) {
      const int rt = tile % p.row_tiles;
      const int tt = tile / p.row_tiles;
      const int buf = lt & 1;
      const uint32_t acc_phase = (lt >> 1) & 1;
      if (!mbar_wait(&sm.accfull[buf], acc_phase, abort_flag, p.status)) break;
      tc_fence_after();
      const int64_t row = static_cast<int64_t>(rt) * kTileRows + q * 32 + lane;
      const bool row_ok = row < rows_total;
      const int t0 = tt * p.bt;
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(buf * p.bt);
      const int nchunks = p.bt / 32 > 0 ? p.bt / 32 : 1;
      for (int c = 0; c < nchunks; ++c) {
        uint32_t v[32];
        tmem_ld32(taddr + static_cast<uint32_t>(c * 32), v);
        tmem_ld_wait();
        if (c == nchunks - 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&sm.accempty[buf]);
        }
        const int cw = p.bt < 32 ? p.bt : 32;
        if (row_ok) {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int64_t t = t0 + c * 32 + j;
            if (j < cw && t < p.M) {
              const __nv_bfloat16 h = __float2bfloat16_rn(__uint_as_float(v[j]));
              p.out[t * ld + row] = __bfloat16_as_ushort(h);
            }
          }
        }
      }
    }
  } else if (warp >= 8) {
    // ---------------- dequantisers ----------------
    const int i = threadIdx.x - 256;        // 0..255
    const int blk = i >> 1;                 // block slot inside the stage
    const int half = i & 1;                 // which 32 weights of the block
    // FWD: slot = weight row n (0..127), one block per row per stage.
    // DX:  slot = (column block kb in 0..1) * 64 + weight row n (0..63).
    const int n_loc = dx ? (blk & 63) : blk;
    const int kb_loc = dx ? (blk >> 6) : 0;
    const uint32_t code_off = dx ? static_cast<uint32_t>(n_loc * 64 + kb_loc * 32 + half * 16)
                                 : static_cast<uint32_t>(n_loc * 32 + half * 16);
    const uint32_t out_row = dx ? static_cast<uint32_t>(kb_loc * 8192 + (n_loc >> 3) * 1024 + (n_loc & 7) * 128)
                                : static_cast<uint32_t>((n_loc >> 3) * 1024 + (n_loc & 7) * 128);
    const uint32_t sw = static_cast<uint32_t>(n_loc & 7);
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
      const int rt = tile % p.row_tiles;
      // scale index for main-loop step k (returns q8 = 0 outside the matrix)
      auto scale_at = [&](int k, uint32_t &q8, float &d) {
        int64_t n, kb;
        if (!dx) { n = static_cast<int64_t>(rt) * kTileRows + n_loc; kb = k; }
        else     { n = static_cast<int64_t>(k) * kKStage + n_loc; kb = static_cast<int64_t>(rt) * 2 + kb_loc; }
        q8 = 0;
        d = 0.f;
        if (k < p.nk && n < p.N && kb < kb_row) {
          const int64_t b = n * kb_row + kb;
          q8 = __ldg(p.scale8 + b);
          d = __ldg(p.scale2 + (b >> 8));
        }
      };
      uint32_t q0, q1, q2;
      float d0, d1, d2;
      scale_at(0, q0, d0);
      scale_at(1, q1, d1);
      for (int k = 0; k < iters; ++k) {
        scale_at(k + 2, q2, d2);   // prefetch two steps ahead
        if (!mbar_wait(&sm.full[stage], phase, abort_flag, p.status)) { ok = false; break; }
        if (k < p.nk) {
          const uint8_t *c = sm.c + static_cast<size_t>(stage) * kCodeTileBytes;
          uint8_t *a = sm.a + static_cast<size_t>(stage) * kATileBytes + out_row;
          const uint4 cw = *reinterpret_cast<const uint4 *>(c + code_off);
          const Nf4Table t = make_table(block_scale(q0, d0));
          const uint32_t w[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            uint32_t o[4];
            expand8(t, w[j], o);
            const uint32_t chunk = (static_cast<uint32_t>(half * 4 + j) ^ sw) * 16u;
            *reinterpret_cast<uint4 *>(a + chunk) = make_uint4(o[0], o[1], o[2], o[3]);
          }
          fence_proxy_async_smem();
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.afull[stage]);
        q0 = q1; d0 = d1;
        q1 = q2; d1 = d2;
        if (++stage == p.stages) { stage = 0; phase ^= 1; }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, tmem_cols);
  }
}

CUtensorMapSwizzle lora_swizzle(int r_pad) {
  return r_pad == 16 ? CU_TENSOR_MAP_SWIZZLE_32B
                     : (r_pad == 32 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B);
}

}  // namespace

// Host-side tensor-map encoder (driver entry point, resolved once).
bool encode_2d(CUtensorMap *map, CUtensorMapDataType dtype, const void *base, uint64_t inner,
               uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
               CUtensorMapSwizzle swizzle);

size_t fused_gemm_smem_bytes(int bt, int stages) {
  return 1024 /* alignment slack */ + static_cast<size_t>(stages) * (kATileBytes + bt * 128u + kCodeTileBytes) +
         static_cast<size_t>(3 * stages + 5) * 8 + 16;
}

static int pick_stages(int bt) {
  const size_t budget = 227 * 1024;
  int s = 8;
  while (s > 2 && fused_gemm_smem_bytes(bt, s) > budget) --s;
  return s;
}

cudaError_t launch_fused_gemm(const GemmArgs &a, cudaStream_t st) {
  GemmParams p{};
  p.scale8 = a.scale8;
  p.scale2 = a.scale2;
  p.out = a.out;
  p.status = a.dev_status;
  p.N = a.N;
  p.K = a.K;
  p.M = a.M;
  p.mode = a.mode;
  int bt = 256;
  if (a.M <= 16) bt = 16;
  else if (a.M <= 32) bt = 32;
  else if (a.M <= 64) bt = 64;
  else if (a.M <= 128) bt = 128;
  p.bt = bt;
  p.stages = pick_stages(bt);
  p.r_pad = a.r <= 16 ? 16 : (a.r <= 32 ? 32 : 64);
  const int64_t rows = a.mode == 0 ? a.N : a.K;         // UMMA M extent
  p.row_tiles = static_cast<int>((rows + kTileRows - 1) / kTileRows);
  p.tok_tiles = static_cast<int>((a.M + bt - 1) / bt);
  p.nk = static_cast<int>(a.mode == 0 ? a.K / kKStage : (a.N + kKStage - 1) / kKStage);

  CUtensorMap tm_act, tm_codes, tm_lw, tm_la;
  const CUtensorMapSwizzle lsw = lora_swizzle(p.r_pad);
  bool ok = true;
  if (a.mode == 0) {
    ok &= encode_2d(&tm_act, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.act, a.K, a.M, a.K * 2, 64, bt,
                    CU_TENSOR_MAP_SWIZZLE_128B);
    ok &= encode_2d(&tm_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.codes, a.K / 2, a.N, a.K / 2, 32,
                    kTileRows, CU_TENSOR_MAP_SWIZZLE_NONE);
    ok &= encode_2d(&tm_lw, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.lora_w, a.r, a.N, a.r * 2, p.r_pad,
                    kTileRows, lsw);
  } else {
    ok &= encode_2d(&tm_act, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.act, a.N, a.M, a.N * 2, 64, bt,
                    CU_TENSOR_MAP_SWIZZLE_128B);
    ok &= encode_2d(&tm_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.codes, a.K / 2, a.N, a.K / 2, 64,
                    64, CU_TENSOR_MAP_SWIZZLE_NONE);
    ok &= encode_2d(&tm_lw, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.lora_w, a.K, a.r, a.K * 2, 64,
                    p.r_pad, CU_TENSOR_MAP_SWIZZLE_128B);
  }
  ok &= encode_2d(&tm_la, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.lora_act, a.r, a.M, a.r * 2, p.r_pad, bt,
                  lsw);
  if (!ok) return cudaErrorInvalidValue;

  const size_t smem = fused_gemm_smem_bytes(bt, p.stages);
  cudaError_t e = cudaFuncSetAttribute(fused_nf4_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int ntiles = p.row_tiles * p.tok_tiles;
  const int sms = device_sm_count();
  const int grid = ntiles < sms ? ntiles : sms;
  fused_nf4_gemm_kernel<<<grid, kThreads, smem, st>>>(tm_act, tm_codes, tm_lw, tm_la, p);
  return cudaGetLastError();
}

}  // namespace qlora
