// Forward of the QLoRA linear for a handful of tokens (M <= 16):
//   Y[t, n] = sum_k X[t, k] W'[n, k] + sum_j sU[t, j] Bl[n, j]
// ("QLoRA, in depth", section "The mechanism in brief": y = W x + (alpha/r) B A
// x with W dequantised to bf16; "QLoRA and Fine-Tuning on One Consumer GPU",
// section "The idea in one line": each weight is dequantised only for the
// moment it is used).
//
// With so few tokens the product is bound by reading the packed weight
// (0.516 B per weight), so the design aims at streaming W at HBM speed with as
// much independent work per SM as possible, not at tensor-core throughput:
//
// * Codes go from global memory straight into registers and are dequantised
//   into the A fragments of the warp-level MMA (m16n8k16, bf16 in, fp32
//   accumulate): no shared-memory staging of W', no barriers between
//   producer and consumer roles. The weight value is exactly the W' of the
//   format, bf16_rn(level * fp32(q8 * d)).
// * Thread (g, c) of a warp (g = lane / 4, c = lane % 4) owns weight rows g and
//   g + 8 of the warp's 16-row tile and, within a span of four NF4 blocks (256
//   K), the whole block c: 32 bytes of codes per row, one table per row and
//   block. The K order inside an MMA step is permuted accordingly (step
//   2i + h takes K = 64c + 8i + 4h + {0..3} from thread c), and the
//   activations are read with the same permutation, so the sum is unchanged.
// * X (the CTA's K range, all tokens) sits in shared memory in a padded layout
//   that makes the 16-byte fragment loads bank-conflict free.
// * K is split over the CTAs of a thread-block cluster (up to 8); each CTA
//   leaves its fp32 partial tile in shared memory and the cluster adds the
//   partials through distributed shared memory in rank order, then adds the
//   LoRA term in fp32 and stores bf16 (deterministic, no workspace).
//
// * Given the adapter A instead of sU, the kernel also computes the LoRA
//   down-projection sU = bf16(s X A^T) itself. A cluster is cx row groups x cs
//   K chunks; each CTA forms X A^T over its K chunk's spans congruent to its
//   row-group index modulo cx (the same fragment scheme, A read from global
//   memory in place of W', the activations already in shared memory), so a
//   cluster reads A once; the partials are added over the whole cluster and
//   rounded once; one CTA writes sU out for the backward. A few-token forward
//   is then a single launch.
//
// CTA: 8 warps = 4 row tiles of 16 rows x 2 warps that split the CTA's spans.
#include "qlora_device.cuh"

namespace qlora {
namespace {

constexpr int kWarps = 8;
constexpr int kRowsPerCta = 64;
constexpr int kTokStride = 144;   // bytes per token row of one 64-K block in smem (128 + 16 pad)

// bytes per 64-K block of the smem activation tile for mp (8 or 16) tokens;
// congruent to 32 mod 128 so that threads c = 0..3 land on distinct banks
__host__ __device__ constexpr uint32_t block_stride(int mp) { return static_cast<uint32_t>(mp * kTokStride + 32); }

__device__ __forceinline__ uint4 ldg_nc_v4(const void *p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// 16-byte asynchronous copy global -> shared; src_bytes = 0 writes zeros
// (the global address is then not read).
__device__ __forceinline__ void cp_async_16(uint32_t saddr, const void *gptr, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(saddr), "l"(gptr), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

__device__ __forceinline__ uint4 lds_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

// The codes and block constants one thread needs for one span: rows g and
// g + 8, block c of the span.
struct SpanCodes {
  uint4 w0a, w0b, w1a, w1b;
  uint32_t q0, q1;
  float d0, d1;
};

__device__ __forceinline__ void load_span(SpanCodes &s, const uint8_t *__restrict__ codes,
                                          const uint8_t *__restrict__ scale8, const float *__restrict__ scale2,
                                          int64_t n0, int64_t K, int64_t cb0, int nb_loc, int nspan, int sp,
                                          int c) {
  const int lb = sp * 4 + c;
  if (sp < nspan && lb < nb_loc) {
    const int64_t b = cb0 + lb, kblocks = K / 64;
    const uint8_t *p0 = codes + n0 * (K / 2) + b * 32;
    const uint8_t *p1 = p0 + 8 * (K / 2);
    s.w0a = ldg_nc_v4(p0);
    s.w0b = ldg_nc_v4(p0 + 16);
    s.w1a = ldg_nc_v4(p1);
    s.w1b = ldg_nc_v4(p1 + 16);
    const int64_t i0 = n0 * kblocks + b, i1 = i0 + 8 * kblocks;
    s.q0 = __ldg(scale8 + i0);
    s.q1 = __ldg(scale8 + i1);
    s.d0 = __ldg(scale2 + (i0 >> 8));
    s.d1 = __ldg(scale2 + (i1 >> 8));
  } else {
    // outside the K range: zero weights (the activations there are zero too)
    s.w0a = s.w0b = s.w1a = s.w1b = make_uint4(0, 0, 0, 0);
    s.q0 = s.q1 = 0;
    s.d0 = s.d1 = 0.f;
  }
}

template <int NTOK>
__device__ __forceinline__ void compute_span(const SpanCodes &s, float (&d)[NTOK][4], uint32_t xrow) {
  const Nf4Table t0 = make_table(block_scale(s.q0, s.d0)), t1 = make_table(block_scale(s.q1, s.d1));
  const uint32_t w0[8] = {s.w0a.x, s.w0a.y, s.w0a.z, s.w0a.w, s.w0b.x, s.w0b.y, s.w0b.z, s.w0b.w};
  const uint32_t w1[8] = {s.w1a.x, s.w1a.y, s.w1a.z, s.w1a.w, s.w1b.x, s.w1b.y, s.w1b.z, s.w1b.w};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    uint32_t r0[4], r1[4];
    expand8(t0, w0[i], r0);
    expand8(t1, w1[i], r1);
#pragma unroll
    for (int u = 0; u < NTOK; ++u) {
      // X[token g + 8u][64 lb + 8i .. + 7] as four bf16 pairs
      const uint4 bx = lds_v4(xrow + static_cast<uint32_t>(u * 8 * kTokStride + i * 16));
      const uint32_t a_lo[4] = {r0[0], r1[0], r0[1], r1[1]};
      const uint32_t a_hi[4] = {r0[2], r1[2], r0[3], r1[3]};
      mma_16816(d[u], a_lo, bx.x, bx.y);
      mma_16816(d[u], a_hi, bx.z, bx.w);
    }
  }
}

template <int NTOK>   // token tiles of 8: 1 (M <= 8) or 2 (M <= 16)
__global__ void __launch_bounds__(kWarps * 32, 2)
    nf4_gemv_fwd_kernel(const uint8_t *__restrict__ codes, const uint8_t *__restrict__ scale8,
                        const float *__restrict__ scale2, int64_t N, int64_t K, int M,
                        const uint16_t *__restrict__ X, const uint16_t *__restrict__ Bl,
                        const uint16_t *__restrict__ sU, const uint16_t *__restrict__ Al, float s_lora,
                        uint16_t *__restrict__ sU_out, int r, int blocks_per_cta, int cx,
                        uint16_t *__restrict__ Y) {
  constexpr int mp = 8 * NTOK;
  constexpr uint32_t bstride = block_stride(mp);
  extern __shared__ __align__(16) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;
  // cluster = cx row groups (x) by csize K chunks (y); rank = x + y * cx
  const uint32_t csize = gridDim.y;
  const uint32_t cxu = static_cast<uint32_t>(cx);
  const uint32_t my_x = blockIdx.x % cxu;
  const uint32_t rank = my_x + blockIdx.y * cxu;
  const int64_t row0 = static_cast<int64_t>(blockIdx.x) * kRowsPerCta;
  const int64_t kblocks = K / 64;
  const int64_t cb0 = static_cast<int64_t>(blockIdx.y) * blocks_per_cta;
  const int64_t cb1 = cb0 + blocks_per_cta < kblocks ? cb0 + blocks_per_cta : kblocks;
  const int nb_loc = cb1 > cb0 ? static_cast<int>(cb1 - cb0) : 0;
  const int nspan = (nb_loc + 3) / 4;

  uint8_t *xs = smem;                                                   // [4 * nspan blocks][mp][144 B]
  float *red = reinterpret_cast<float *>(smem + static_cast<size_t>(4 * nspan) * bstride);   // [2][64][mp]
  float *sum = red + 2 * kRowsPerCta * mp;                                                // [64][mp]
  float *uslot = sum + kRowsPerCta * mp;   // [8 parts][64 j][mp]: X A^T partials of this CTA's warps
  float *usum = uslot + 8 * 64 * mp;       // [64 j][mp]: this CTA's X A^T over its K range
  float *su_s = usum + 64 * mp;            // [mp][64 j]: bf16(s X A^T) of all tokens, as float

  // Warp (rt, half) takes the spans half, half + 2, ... of its 16-row tile.
  // Its first two spans are requested before anything else so that their
  // latency overlaps the activation fill and the adapter projection; then a
  // third; afterwards a span is requested as soon as its registers are
  // consumed (three spans per warp in flight).
  const int rt = warp >> 1, half = warp & 1;
  const int64_t n0 = row0 + rt * 16 + g;
  const bool rows_ok = row0 + rt * 16 < N;   // N % 16 == 0: a row tile is all in or all out
  const int nsp = rows_ok ? nspan : 0;
  SpanCodes sa, sb, sc;
  load_span(sa, codes, scale8, scale2, n0, K, cb0, nb_loc, nsp, half, c);
  load_span(sb, codes, scale8, scale2, n0, K, cb0, nb_loc, nsp, half + 2, c);

  // ---- activations of this K range -> shared memory (zero beyond M and K),
  // every 16-byte piece requested at once ----
  {
    const int pieces = 4 * nspan * mp * 8;
    const uint32_t xs_s = smem_u32(xs);
    for (int i = threadIdx.x; i < pieces; i += blockDim.x) {
      const int piece = i & 7;
      const int t = (i >> 3) % mp;
      const int lb = (i >> 3) / mp;
      const bool in = t < M && lb < nb_loc;
      const uint16_t *src = in ? X + static_cast<int64_t>(t) * K + (cb0 + lb) * 64 + piece * 8 : X;
      cp_async_16(xs_s + static_cast<uint32_t>(lb) * bstride + static_cast<uint32_t>(t * kTokStride + piece * 16), src,
                  in ? 16u : 0u);
    }
    cp_async_wait_all();
  }
  __syncthreads();

  const uint32_t xs_base = smem_u32(xs) + static_cast<uint32_t>(g * kTokStride + c * bstride);
  const int jt_n = (r + 15) / 16;            // 16-row tiles of the adapter rank
  if (Al != nullptr) {
    // partial U[j, t] = sum over this CTA's K of A[j, k] X[t, k], while the
    // first weight spans are in flight: warp w takes
    // rank tile w % jt_n and the spans congruent to w / jt_n modulo 8 / jt_n
    const int parts = kWarps / jt_n;
    if (warp < parts * jt_n) {
      const int jt = warp % jt_n, part = warp / jt_n;
      const int j0 = jt * 16 + g, j1 = j0 + 8;
      float ud[NTOK][4];
#pragma unroll
      for (int u = 0; u < NTOK; ++u) ud[u][0] = ud[u][1] = ud[u][2] = ud[u][3] = 0.f;
      for (int sp = static_cast<int>(my_x) + part * cx; sp < nspan; sp += parts * cx) {
        const int lb = sp * 4 + c;
        const bool valid = lb < nb_loc;
        const uint16_t *a0 = Al + static_cast<int64_t>(j0) * K + (cb0 + lb) * 64;
        const uint16_t *a1 = Al + static_cast<int64_t>(j1) * K + (cb0 + lb) * 64;
        const uint32_t xrow = xs_base + static_cast<uint32_t>(4 * sp) * bstride;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint4 ra = valid && j0 < r ? __ldg(reinterpret_cast<const uint4 *>(a0 + 8 * i)) : make_uint4(0, 0, 0, 0);
          const uint4 rb = valid && j1 < r ? __ldg(reinterpret_cast<const uint4 *>(a1 + 8 * i)) : make_uint4(0, 0, 0, 0);
#pragma unroll
          for (int u = 0; u < NTOK; ++u) {
            const uint4 bx = lds_v4(xrow + static_cast<uint32_t>(u * 8 * kTokStride + i * 16));
            const uint32_t a_lo[4] = {ra.x, rb.x, ra.y, rb.y};
            const uint32_t a_hi[4] = {ra.z, rb.z, ra.w, rb.w};
            mma_16816(ud[u], a_lo, bx.x, bx.y);
            mma_16816(ud[u], a_hi, bx.z, bx.w);
          }
        }
      }
#pragma unroll
      for (int u = 0; u < NTOK; ++u) {
        float *dst = uslot + (part * 64 + jt * 16) * mp + 8 * u + 2 * c;
        dst[g * mp] = ud[u][0];
        dst[g * mp + 1] = ud[u][1];
        dst[(g + 8) * mp] = ud[u][2];
        dst[(g + 8) * mp + 1] = ud[u][3];
      }
    }
  }

  load_span(sc, codes, scale8, scale2, n0, K, cb0, nb_loc, nsp, half + 4, c);

  float d[NTOK][4];
#pragma unroll
  for (int u = 0; u < NTOK; ++u) d[u][0] = d[u][1] = d[u][2] = d[u][3] = 0.f;
  for (int sp = half; sp < nsp; sp += 6) {
    compute_span<NTOK>(sa, d, xs_base + static_cast<uint32_t>(4 * sp) * bstride);
    load_span(sa, codes, scale8, scale2, n0, K, cb0, nb_loc, nsp, sp + 6, c);
    if (sp + 2 >= nsp) break;
    compute_span<NTOK>(sb, d, xs_base + static_cast<uint32_t>(4 * (sp + 2)) * bstride);
    load_span(sb, codes, scale8, scale2, n0, K, cb0, nb_loc, nsp, sp + 8, c);
    if (sp + 4 >= nsp) break;
    compute_span<NTOK>(sc, d, xs_base + static_cast<uint32_t>(4 * (sp + 4)) * bstride);
    load_span(sc, codes, scale8, scale2, n0, K, cb0, nb_loc, nsp, sp + 10, c);
  }

  // ---- reduce: the two warps of a row tile, then the cluster's CTAs ----
  // D fragment: d[u][0..1] = rows g, tokens 8u + 2c, 2c + 1; d[u][2..3] = row g + 8
#pragma unroll
  for (int u = 0; u < NTOK; ++u) {
    float *dst = red + (half * kRowsPerCta + rt * 16) * mp + 8 * u + 2 * c;
    dst[g * mp] = d[u][0];
    dst[g * mp + 1] = d[u][1];
    dst[(g + 8) * mp] = d[u][2];
    dst[(g + 8) * mp + 1] = d[u][3];
  }
  __syncthreads();
  for (int i = threadIdx.x; i < kRowsPerCta * mp; i += blockDim.x) sum[i] = red[i] + red[kRowsPerCta * mp + i];
  if (Al != nullptr) {
    const int parts = kWarps / jt_n;
    for (int i = threadIdx.x; i < jt_n * 16 * mp; i += blockDim.x) {
      float u = 0.f;
      for (int q = 0; q < parts; ++q) u += uslot[q * 64 * mp + i];
      usum[i] = u;
    }
  }
  cluster_sync_all();

  // the LoRA down-projection of all tokens, added over the cluster in rank order
  if (Al != nullptr) {
    const uint32_t usum_addr = smem_u32(usum);
    for (int i = threadIdx.x; i < M * r; i += blockDim.x) {
      const int t = i / r, j = i % r;
      const uint32_t off = static_cast<uint32_t>((j * mp + t) * 4);
      float u = 0.f;
      for (uint32_t q = 0; q < csize * cxu; ++q) u += ld_dsmem_f32(mapa_shared(usum_addr + off, q));
      const __nv_bfloat16 v = __float2bfloat16_rn(s_lora * u);
      su_s[t * 64 + j] = __bfloat162float(v);
      if (sU_out != nullptr && blockIdx.x == 0 && rank == 0) sU_out[static_cast<int64_t>(t) * r + j] = __bfloat16_as_ushort(v);
    }
  } else {
    for (int i = threadIdx.x; i < M * r; i += blockDim.x) {
      const int t = i / r, j = i % r;
      su_s[t * 64 + j] = __uint_as_float(static_cast<uint32_t>(sU[static_cast<int64_t>(t) * r + j]) << 16);
    }
  }
  __syncthreads();

  // K chunk q of a row group finishes rows [q * 64 / csize, (q + 1) * 64 / csize)
  const int rows_per = kRowsPerCta / static_cast<int>(csize);
  const int rl0 = static_cast<int>(blockIdx.y) * rows_per;
  const uint32_t sum_addr = smem_u32(sum);
  for (int i = threadIdx.x; i < rows_per * M; i += blockDim.x) {
    const int t = i / rows_per, rl = rl0 + i % rows_per;
    const int64_t n = row0 + rl;
    if (n >= N) continue;
    const uint32_t off = static_cast<uint32_t>((rl * mp + t) * 4);
    float y = 0.f;
    for (uint32_t q = 0; q < csize; ++q) y += ld_dsmem_f32(mapa_shared(sum_addr + off, my_x + q * cxu));
    float l = 0.f;
    const uint16_t *brow = Bl + n * r;
    const float *urow = su_s + t * 64;
    for (int j = 0; j < r; ++j) l = fmaf(urow[j], __uint_as_float(static_cast<uint32_t>(brow[j]) << 16), l);
    Y[static_cast<int64_t>(t) * N + n] = __bfloat16_as_ushort(__float2bfloat16_rn(y + l));
  }
  cluster_sync_all();   // no CTA leaves while another still reads its partials
}

}  // namespace

namespace {
size_t gemv_smem_bytes(int64_t K, int64_t M, int cs) {
  const int64_t kblocks = K / 64;
  const int64_t bpc = (kblocks + cs - 1) / cs;
  const int mp = M <= 8 ? 8 : 16;
  return static_cast<size_t>(4 * ((bpc + 3) / 4)) * block_stride(mp) +
         static_cast<size_t>(3 * kRowsPerCta * mp + 8 * 64 * mp + 64 * mp + mp * 64) * 4;
}

// Cluster size (K split) for an [N, K] weight and M tokens, or 0 when the
// shape does not suit this kernel. K is split while the grid still fits in one
// wave of two CTAs per SM and every CTA keeps at least two spans of K (up to a
// cluster of 8); then further if the activation tile does not fit in shared
// memory.
int gemv_cluster(int64_t N, int64_t K, int64_t M) {
  if (M < 1 || M > 16 || N < 1 || K < 64) return 0;
  const int64_t row_groups = (N + kRowsPerCta - 1) / kRowsPerCta;
  const int64_t kblocks = K / 64;
  const int sms = device_sm_count();
  int cs = 1;
  while (cs < 8 && row_groups * cs * 2 <= 2 * sms && kblocks >= 8 * cs) cs *= 2;
  while (cs < 8 && gemv_smem_bytes(K, M, cs) > 200 * 1024) cs *= 2;
  return gemv_smem_bytes(K, M, cs) <= 200 * 1024 ? cs : 0;
}
}  // namespace

bool gemv_fwd_supported(int64_t N, int64_t K, int64_t M) { return gemv_cluster(N, K, M) > 0; }

cudaError_t launch_nf4_gemv_fwd(const uint8_t *codes, const uint8_t *scale8, const float *scale2, int64_t N,
                                int64_t K, int64_t M, const uint16_t *X, const uint16_t *Bl, const uint16_t *sU,
                                const uint16_t *Al, float s, uint16_t *sU_out, int r, uint16_t *Y,
                                cudaStream_t st) {
  if ((sU == nullptr) == (Al == nullptr)) return cudaErrorInvalidValue;
  const int cs = gemv_cluster(N, K, M);
  if (cs == 0) return cudaErrorInvalidValue;
  // with the adapter's down-projection inside, cx row groups share one
  // cluster (and one read of A); the grid is padded to a multiple of cx
  int cx = 1;
  const int64_t rg_real = (N + kRowsPerCta - 1) / kRowsPerCta;
  if (Al != nullptr)
    while (cx * 2 * cs <= 8 && cx * 2 <= rg_real) cx *= 2;
  const int64_t row_groups = (rg_real + cx - 1) / cx * cx;
  const int bpc = static_cast<int>((K / 64 + cs - 1) / cs);
  const int ntok = M <= 8 ? 1 : 2;
  const size_t smem = gemv_smem_bytes(K, M, cs);
  const void *fn = ntok == 1 ? reinterpret_cast<const void *>(nf4_gemv_fwd_kernel<1>)
                             : reinterpret_cast<const void *>(nf4_gemv_fwd_kernel<2>);
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(row_groups), static_cast<unsigned>(cs), 1);
  cfg.blockDim = dim3(kWarps * 32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(cx);
  attr[0].val.clusterDim.y = static_cast<unsigned>(cs);
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int Mi = static_cast<int>(M), bpc_arg = bpc;
  void *args[] = {&codes, &scale8, &scale2, &N, &K, &Mi, &X, &Bl, &sU, &Al, &s, &sU_out, &r, &bpc_arg, &cx, &Y};
  return cudaLaunchKernelExC(&cfg, fn, args);
}

}  // namespace qlora
