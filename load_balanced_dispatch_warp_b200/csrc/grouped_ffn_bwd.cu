// Backward pass of the MoE layer's expert path (sm_100a).
//
// The MoonEP news article (paragraph 3): the duplicated experts' "gradients get reduced
// back home during the backward pass".  With dy = dLoss/dy for every row of the per-rank
// buffers (moe_combine_backward), each plan group (rows r0..r0+n of one rank, expert e)
// runs the chain rule of its SwiGLU expert (forward g = X W1^T, u = X W3^T,
// h = silu(g) u, y = h W2^T):
//   dH  = dY W2                    [rows, F]   GEMM, bf16 x bf16 -> fp32
//   dG  = dH * u * silu'(g),  dU = dH * silu(g)
//                                  [rows, F]   the gate/up GEMM re-run on the rows, with
//                                              an epilogue that reads dH (no saved g, u)
//   dX  = dG W1 + dU W3            [rows, d]   GEMM over K = 2F, bf16
//   dW2[e] += dY^T h, dW1[e] += dG^T X, dW3[e] += dU^T X
//                                              GEMMs over the rows of every group of
//                                              expert e -- home and replica groups in one
//                                              accumulator: the reduction back home
// All GEMMs run on one persistent tcgen05 kernel (TMA-fed 4-stage ring, TMEM double
// buffer, one MMA thread, four epilogue warps) with three epilogues, in bf16: dY is bf16
// because gate * dout spans the gates' range (fp16 would lose small gates to subnormals),
// and the fp16 operand it meets in dH (W2) is converted to bf16 by a transpose.  The dX
// GEMM reads W1 and W3 as they are stored (MN-major B operand).  The weight-gradient
// GEMMs read dY, h, dG | dU and X as the forward and the other GEMMs left them, row-major
// [rows, columns] with the K dimension (rows) outermost: both operands MN-major.  Their K
// steps walk each group of the expert 64 rows at a time; in a group's last, partial step
// the rows past the group's end belong to the next group, and the MMA warp zeroes them in
// the A tile (whole 128-byte rows of the swizzled box) before the MMAs read it.  h is
// recomputed in the SwiGLU-backward epilogue (silu(g) * u from the re-run gate/up GEMM)
// and stored as bf16, the type dY needs its partner to have.
#include <cuda.h>

#include "rows.cuh"

namespace moe {
namespace {

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int UMMA_K = 16;
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;
constexpr int B_BYTES_MAX = 256 * BK * 2;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES_MAX;
constexpr int ACC_COLS = 256;
constexpr int TMEM_COLS = 2 * ACC_COLS;
constexpr int MAX_GROUPS = 4096;
constexpr int BWD_THREADS = 192;
constexpr uint64_t WAIT_LIMIT_NS = 2000000000ull;

enum { EPI_BF16 = 0, EPI_F32 = 1, EPI_SWIGLU_BWD = 2 };

struct BwdArgs {
  const int4* groups;   // plan group records {row_start, rows, expert, weight_ref}
  int G;
  int n_blocks_n;       // output column blocks
  int k_blocks;         // K / BK (row tiles)
  int bn_out;           // output columns per tile
  int mma_n;            // N of the MMA (256 with two B halves for the SwiGLU backward)
  int rows_per_expert;  // rows of one expert in the B tensor (row tiles)
  int out_ld;           // columns of the output tensor
  int bf16;             // operand type: 1 bf16, 0 fp16
  int kb_split;         // B read MN-major: K steps below it from tm_b0, the rest from tm_b1
  int e_home;           // row tiles: experts of the home maps (tm_b*); a group whose expert
                        // index is e_home or above reads pool slot index - e_home from tm_p*
  void* out;
  int32_t* err;
  // SwiGLU backward epilogue: reads dH [rows, F] fp32, writes dG | dU into dGU [rows, 2F]
  // and h = silu(g) * u into hb [rows, F] (bf16)
  const float* dh;
  __nv_bfloat16* dgu;
  __nv_bfloat16* hb;
  int F;
  // weight-gradient tiles: (expert, m block, n block), K over the rows of the expert's
  // groups; A and B are row-major activations read MN-major (column a_row, b_row)
  const int* seg_off;   // [E+1]
  const int2* segs;     // {row_start, rows} of each group of the expert
  int m_blocks;
  int a_row_base;
  int64_t out_expert_stride;
  int E;
};

// ------------------------------------------------------------------- PTX wrappers
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait (about 2 s of %globaltimer); false if it ran out or another role aborted.
__device__ __noinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                       int32_t* err) {
  if (mbar_try(bar, parity)) return true;
  uint64_t t0 = 0;
  for (uint32_t it = 1;; ++it) {
    if (mbar_try(bar, parity)) return true;
    if ((it & 255u) == 0) {
      if (*abort_flag) return false;
      const uint64_t now = globaltimer();
      if (t0 == 0) {
        t0 = now;
      } else if (now - t0 > WAIT_LIMIT_NS) {
        *abort_flag = 1;
        atomicOr(err, MOE_DERR_TIMEOUT);
        return false;
      }
    }
  }
}
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}
// shared -> global tile store through the tensor map (bulk group of the issuing thread)
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, uint32_t src, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(x), "r"(y), "r"(src)
      : "memory");
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}
__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
// K-major tile written by TMA with the 128-byte swizzle (8-row atoms 1024 bytes apart).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)1 << 16) |
         ((uint64_t)(1024 >> 4) << 32) | ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}
// MN-major tile written by TMA with the 128-byte swizzle as boxes of 64 K rows x 64 MN
// elements (128-byte rows): 8-row K groups 1024 bytes apart (stride byte offset), 64-element
// MN chunks one box (8 KiB) apart (leading byte offset).  A K step of 16 rows adds 2048
// bytes to the start address.
__device__ __forceinline__ uint64_t sw128_mn_desc(uint32_t saddr) {
  return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)(8192 >> 4) << 16) |
         ((uint64_t)(1024 >> 4) << 32) | ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}
// kind::f16 instruction descriptor: fp32 accumulate, A and B bf16 (1) or fp16 (0), A
// K-major (0) or MN-major (1) at bit 15, B likewise at bit 16, N >> 3 at bits 17-22,
// M >> 4 at bits 24-28.
__device__ __forceinline__ uint32_t make_idesc(int M, int N, bool bf16, bool b_mn,
                                               bool a_mn = false) {
  return (1u << 4) | ((bf16 ? 1u : 0u) << 7) | ((bf16 ? 1u : 0u) << 10) |
         ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}
__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}

// ------------------------------------------------------------------- tiles
struct BTile {
  int a_row;       // first A row
  int valid_rows;  // rows of the block to store
  int b_row;       // first B row
  int n_block;
  int e;               // row tiles: the group's weights inside their tensor; weight-gradient
                       // tiles: the output expert
  bool pool;           // row tiles: B from the pool maps
  int seg_lo, seg_hi;  // weight-gradient tiles: the expert's K segments
  int64_t out_off;     // element offset of the tile's first output row and column
};

template <bool WGRAD>
__device__ __forceinline__ BTile decode(int t, const BwdArgs& a, const int* s_prefix) {
  BTile tl;
  if (WGRAD) {
    const int per = a.m_blocks * a.n_blocks_n;
    const int e = t / per;
    const int rem = t - e * per;
    const int mb = rem / a.n_blocks_n;
    tl.n_block = rem - mb * a.n_blocks_n;
    tl.a_row = a.a_row_base + mb * BM;
    tl.valid_rows = BM;
    tl.b_row = tl.n_block * a.bn_out;
    tl.e = e;
    tl.seg_lo = __ldg(a.seg_off + e);
    tl.seg_hi = __ldg(a.seg_off + e + 1);
    tl.out_off = (int64_t)e * a.out_expert_stride + (int64_t)mb * BM * a.out_ld +
                 (int64_t)tl.n_block * a.bn_out;
  } else {
    const int mt = t / a.n_blocks_n;
    tl.n_block = t - mt * a.n_blocks_n;
    int lo = 0, hi = a.G - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_prefix[mid] <= mt) lo = mid; else hi = mid - 1;
    }
    const int4 g = __ldg(a.groups + lo);
    const int m_local = mt - s_prefix[lo];
    tl.a_row = g.x + m_local * BM;
    tl.valid_rows = min(BM, g.y - m_local * BM);
    // g.z indexes the weights: experts below e_home in the home maps (a replica slot holds
    // its expert's weights bitwise, so on one GPU every group reads the home tensor), the
    // rest in the pool maps (a rank of the expert-parallel layer reads its own slots)
    tl.pool = g.z >= a.e_home;
    tl.e = tl.pool ? g.z - a.e_home : g.z;  // index inside its tensor (home or pool)
    tl.b_row = tl.e * a.rows_per_expert + tl.n_block * a.bn_out;
    tl.seg_lo = tl.seg_hi = 0;
    tl.out_off = (int64_t)tl.a_row * a.out_ld + (int64_t)tl.n_block * a.bn_out;
  }
  return tl;
}

// K steps of a tile, in order, as f(k, valid): row tiles f(kb, BK) for kb = 0..k_blocks-1;
// weight-gradient tiles f(first row, rows of the group in the step) for every 64 rows of
// every group of the expert (valid < BK only in a group's last step).
template <bool WGRAD, class F>
__device__ __forceinline__ bool for_k(const BTile& tl, const BwdArgs& a, F&& f) {
  if (WGRAD) {
    for (int s = tl.seg_lo; s < tl.seg_hi; ++s) {
      const int2 sg = __ldg(a.segs + s);
      for (int r = 0; r < sg.y; r += BK)
        if (!f(sg.x + r, min(BK, sg.y - r))) return false;
    }
  } else {
    for (int kb = 0; kb < a.k_blocks; ++kb)
      if (!f(kb, BK)) return false;
  }
  return true;
}

template <int EPI, bool WGRAD, bool BMN>
__global__ void __launch_bounds__(BWD_THREADS, 1)
    bwd_gemm_kernel(const __grid_constant__ CUtensorMap tm_a,
                    const __grid_constant__ CUtensorMap tm_b0,
                    const __grid_constant__ CUtensorMap tm_b1,
                    const __grid_constant__ CUtensorMap tm_p0,
                    const __grid_constant__ CUtensorMap tm_p1,
                    const __grid_constant__ CUtensorMap tm_o, const BwdArgs args) {
  constexpr bool TWO_B = EPI == EPI_SWIGLU_BWD;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* stage_base = smem;
  // fp32 epilogue: a 32 x 32 staging block per epilogue warp, 1024-byte aligned (the
  // weight-gradient tiles leave it through a TMA store with the 128-byte swizzle)
  float* s_stage = reinterpret_cast<float*>(smem + STAGES * STAGE_BYTES);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES + 4 * 32 * 32 * 4);
  int* s_misc = reinterpret_cast<int*>(bars + 2 * STAGES + 5);
  int* s_prefix = s_misc + 4;
  int* s_scan = s_prefix + MAX_GROUPS + 1;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  volatile int* abort_flag = s_misc + 1;

  if (tid == 0) {
    s_misc[2] = load_err(args.err);
    s_misc[1] = 0;
  }
  __syncthreads();
  if (s_misc[2] != 0) return;

  int total_tiles;
  if (WGRAD) {
    total_tiles = args.E * args.m_blocks * args.n_blocks_n;
  } else {
    for (int g = tid; g < args.G; g += blockDim.x) {
      const int rows = __ldg(&args.groups[g].y);
      s_prefix[g] = rows > 0 ? (rows + BM - 1) / BM : 0;
    }
    __syncthreads();
    const int total_m = block_exclusive_scan(s_prefix, args.G, s_scan);
    if (tid == 0) s_prefix[args.G] = total_m;
    total_tiles = total_m * args.n_blocks_n;
  }

  const uint32_t full0 = smem_u32(bars);
  const uint32_t empty0 = smem_u32(bars + STAGES);
  const uint32_t tfull0 = smem_u32(bars + 2 * STAGES);
  const uint32_t tempty0 = smem_u32(bars + 2 * STAGES + 2);
  const uint32_t drain = smem_u32(bars + 2 * STAGES + 4);
  if (tid == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull0 + 8 * b, 1);
      mbar_init(tempty0 + 8 * b, 4);
    }
    mbar_init(drain, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(s_misc)),
                 "r"(TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = static_cast<uint32_t>(s_misc[0]);
  const uint32_t b_bytes = (uint32_t)args.mma_n * BK * 2;

  if (warp == 0) {
    // ------------------------------------------------------------- TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0, issued_phase = 0;
      for (int t = blockIdx.x; t < total_tiles; t += gridDim.x) {
        const BTile tl = decode<WGRAD>(t, args, s_prefix);
        const bool ok = for_k<WGRAD>(tl, args, [&](int kb, int) {
          if (!mbar_wait(empty0 + 8 * stage, phase ^ 1u, abort_flag, args.err)) return false;
          const uint32_t fb = full0 + 8 * stage;
          const uint32_t sa = smem_u32(stage_base + stage * STAGE_BYTES);
          const uint32_t sb = sa + A_BYTES;
          mbar_expect_tx(fb, A_BYTES + b_bytes);
          if (WGRAD) {
            // kb is the step's first row: boxes of 64 rows x 64 columns of the row-major
            // activations, A columns a_row.. (M), B columns b_row.. (N)
            for (int c = 0; c < BM / 64; ++c)
              tma_load_2d(sa + c * 8192, &tm_a, fb, tl.a_row + c * 64, kb);
            for (int c = 0; c < args.mma_n / 64; ++c)
              tma_load_2d(sb + c * 8192, &tm_b0, fb, tl.b_row + c * 64, kb);
          } else {
            tma_load_2d(sa, &tm_a, fb, kb * BK, tl.a_row);
            if (BMN) {
              // B [N][K] read from a tensor stored K-row major: boxes of 64 K rows x 64 N
              const bool lo = kb < args.kb_split;
              const int krow = tl.e * args.rows_per_expert + (lo ? kb : kb - args.kb_split) * BK;
              const int n0 = tl.n_block * args.bn_out;
              for (int c = 0; c < args.mma_n / 64; ++c)
                tma_load_2d(sb + c * 8192,
                            lo ? (tl.pool ? &tm_p0 : &tm_b0) : (tl.pool ? &tm_p1 : &tm_b1), fb,
                            n0 + c * 64, krow);
            } else {
              tma_load_2d(sb, tl.pool ? &tm_p0 : &tm_b0, fb, kb * BK, tl.b_row);
              if (TWO_B)
                tma_load_2d(sb + (b_bytes >> 1), tl.pool ? &tm_p1 : &tm_b1, fb, kb * BK, tl.b_row);
            }
          }
          issued_mask |= 1u << stage;
          issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
          return true;
        });
        if (!ok) break;
      }
      for (int s = 0; s < STAGES; ++s)
        if (issued_mask & (1u << s)) {
          volatile int no_abort = 0;
          mbar_wait(full0 + 8 * s, (issued_phase >> s) & 1u, &no_abort, args.err);
        }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA issuer
    // Lane 0 issues.  Weight-gradient tiles run the loop on the whole warp: in a group's
    // last, partial K step the warp zeroes the A rows past the group's end (they hold the
    // next group's values) after the TMA has landed and before the MMAs read the stage.
    if (WGRAD || lane == 0) {
      const uint32_t idesc = make_idesc(BM, args.mma_n, args.bf16 != 0, BMN || WGRAD, WGRAD);
      const bool issuer = !WGRAD || lane == 0;
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      for (int t = blockIdx.x; t < total_tiles; t += gridDim.x) {
        const BTile tl = decode<WGRAD>(t, args, s_prefix);
        bool okt = mbar_wait(tempty0 + 8 * acc, acc_phase ^ 1u, abort_flag, args.err);
        if (WGRAD) okt = __all_sync(MOE_FULL_MASK, okt);
        if (!okt) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * ACC_COLS;
        bool first = true;
        const bool ok = for_k<WGRAD>(tl, args, [&](int, int valid) {
          bool okf = mbar_wait(full0 + 8 * stage, phase, abort_flag, args.err);
          if (WGRAD) okf = __all_sync(MOE_FULL_MASK, okf);
          if (!okf) return false;
          tc_fence_after();
          const uint32_t sa = smem_u32(stage_base + stage * STAGE_BYTES);
          const uint32_t sb = sa + A_BYTES;
          if (WGRAD && valid < BK) {
            // K row r of an MN-major box is the 128-byte line at r * 128 (the swizzle only
            // permutes 16-byte chunks inside a line): zero lines valid..63 of both boxes
            uint4* a0 = reinterpret_cast<uint4*>(stage_base + stage * STAGE_BYTES);
            const int n16 = (BK - valid) * 8;
            for (int c = 0; c < BM / 64; ++c)
              for (int i = lane; i < n16; i += 32) a0[c * 512 + valid * 8 + i] = make_uint4(0u, 0u, 0u, 0u);
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
          }
          if (issuer) {
#pragma unroll
            for (int kk = 0; kk < BK / UMMA_K; ++kk)
              tc_mma(d_tmem,
                     WGRAD ? sw128_mn_desc(sa + kk * UMMA_K * 128) : sw128_desc(sa + kk * UMMA_K * 2),
                     (BMN || WGRAD) ? sw128_mn_desc(sb + kk * UMMA_K * 128)
                                    : sw128_desc(sb + kk * UMMA_K * 2),
                     idesc, (first && kk == 0) ? 0u : 1u);
            tc_commit(empty0 + 8 * stage);
          }
          if (WGRAD) __syncwarp();
          first = false;
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
          return true;
        });
        if (!ok) break;
        if (issuer) tc_commit(tfull0 + 8 * acc);
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      }
      if (issuer) {
        tc_commit(drain);
        volatile int no_abort = 0;
        mbar_wait(drain, 0, &no_abort, args.err);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------- epilogue (warps 2-5)
    const int quarter = warp & 3;
    const int r_in = quarter * 32 + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = blockIdx.x; t < total_tiles; t += gridDim.x) {
      const BTile tl = decode<WGRAD>(t, args, s_prefix);
      const bool ok = mbar_wait(tfull0 + 8 * acc, acc_phase, abort_flag, args.err);
      if (!__all_sync(MOE_FULL_MASK, ok)) break;
      tc_fence_after();
      const uint32_t tbase = tmem_base + ((uint32_t)(quarter * 32) << 16) + acc * ACC_COLS;
      const bool valid = r_in < tl.valid_rows;
      const bool empty_k = WGRAD && tl.seg_lo == tl.seg_hi;  // expert without rows: zeros
      if (EPI == EPI_SWIGLU_BWD) {
        const int row = tl.a_row + r_in;
        const int col0 = tl.n_block * 128;
        const float* dhrow = args.dh + (int64_t)row * args.F + col0;
        __nv_bfloat16* grow = args.dgu + (int64_t)row * (2 * args.F) + col0;
#pragma unroll 1
        for (int c = 0; c < 128 / 32; ++c) {
          uint32_t g[32], u[32];
          tmem_ld32(tbase + c * 32, g);
          tmem_ld32(tbase + 128 + c * 32, u);
          tmem_wait_ld();
          if (valid) {
            float dh[32];
            const float4* src = reinterpret_cast<const float4*>(dhrow + c * 32);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const float4 v = __ldg(src + i);
              dh[4 * i] = v.x;
              dh[4 * i + 1] = v.y;
              dh[4 * i + 2] = v.z;
              dh[4 * i + 3] = v.w;
            }
            uint32_t pg[16], pu[16], ph[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              float dgv[2], duv[2], hv[2];
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                const float gv = __uint_as_float(g[2 * i + h]);
                const float uv = __uint_as_float(u[2 * i + h]);
                const float s = 1.0f / (1.0f + __expf(-gv));
                const float dhv = dh[2 * i + h];
                duv[h] = dhv * gv * s;
                dgv[h] = dhv * uv * s * (1.0f + gv * (1.0f - s));
                hv[h] = gv * s * uv;
              }
              pg[i] = pack_bf16(dgv[0], dgv[1]);
              pu[i] = pack_bf16(duv[0], duv[1]);
              ph[i] = pack_bf16(hv[0], hv[1]);
            }
            uint4* dg_dst = reinterpret_cast<uint4*>(grow + c * 32);
            uint4* du_dst = reinterpret_cast<uint4*>(grow + args.F + c * 32);
            uint4* h_dst = reinterpret_cast<uint4*>(args.hb + (int64_t)row * args.F + col0 + c * 32);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              dg_dst[i] = make_uint4(pg[4 * i], pg[4 * i + 1], pg[4 * i + 2], pg[4 * i + 3]);
              du_dst[i] = make_uint4(pu[4 * i], pu[4 * i + 1], pu[4 * i + 2], pu[4 * i + 3]);
              h_dst[i] = make_uint4(ph[4 * i], ph[4 * i + 1], ph[4 * i + 2], ph[4 * i + 3]);
            }
          }
        }
      } else if (EPI == EPI_F32) {
        // Each 32-row x 32-column block goes through shared memory so that one store
        // instruction writes four whole 128-byte row segments (lanes 8i..8i+7 one row)
        // instead of 16 bytes in each of 32 rows.  16-byte chunk j of staged row r sits at
        // chunk j ^ (r % 8): the row-per-lane writes and the segment-per-8-lanes reads are
        // both free of bank conflicts.
        // Weight-gradient tiles are whole 128 x N blocks of the output: each staged block,
        // laid out as the 128-byte swizzle places it, leaves through one TMA store issued by
        // lane 0 (the copy engine moves the 4 KiB while the warp stages the next block).
        float* stg = s_stage + (warp - 2) * 1024;
        const int sr = lane >> 3;  // row of this lane within each group of four
        const int sq = lane & 7;   // its 16-byte chunk of the 128-byte segment
        const int rows_here = tl.valid_rows - quarter * 32;
        float* obase = static_cast<float*>(args.out) + tl.out_off +
                       (int64_t)(quarter * 32) * args.out_ld;
        const int o_row = WGRAD ? (int)(tl.out_off / args.out_ld) + quarter * 32 : 0;
        const int o_col = WGRAD ? (int)(tl.out_off % args.out_ld) : 0;
#pragma unroll 1
        for (int c = 0; c < args.bn_out / 32; ++c) {
          uint32_t v[32];
          if (!empty_k) {
            tmem_ld32(tbase + c * 32, v);
            tmem_wait_ld();
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = 0u;
          }
          // the previous block's reads of the staging block are done (TMA: its store has
          // read shared memory)
          if (WGRAD && lane == 0) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
          __syncwarp();
#pragma unroll
          for (int j = 0; j < 8; ++j)
            *reinterpret_cast<float4*>(stg + lane * 32 + ((j ^ (lane & 7)) << 2)) =
                make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]),
                            __uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3]));
          if (WGRAD) {
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
            if (lane == 0) tma_store_2d(&tm_o, smem_u32(stg), o_col + c * 32, o_row);
          } else {
            __syncwarp();
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const int r = 4 * i + sr;
              const float4 val =
                  *reinterpret_cast<const float4*>(stg + r * 32 + ((sq ^ (r & 7)) << 2));
              if (r < rows_here)
                *reinterpret_cast<float4*>(obase + (int64_t)r * args.out_ld + c * 32 + sq * 4) =
                    val;
            }
          }
        }
      } else {
        uint16_t* orow = static_cast<uint16_t*>(args.out) + tl.out_off + (int64_t)r_in * args.out_ld;
#pragma unroll 1
        for (int c = 0; c < args.bn_out / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(tbase + c * 32, v);
          tmem_wait_ld();
          uint32_t p[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) p[i] = pack_bf16(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
          if (valid) {
            uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
            for (int i = 0; i < 4; ++i) dst[i] = make_uint4(p[4 * i], p[4 * i + 1], p[4 * i + 2], p[4 * i + 3]);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty0 + 8 * acc);
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
    // every TMA store of this warp has finished before its staging block goes away
    if (EPI == EPI_F32 && WGRAD && lane == 0)
      asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(TMEM_COLS)
                 : "memory");
  }
}

// ------------------------------------------------------------------- helpers
// Per expert, the list of its groups' row ranges {row_start, rows} in group-table order
// (home and replica groups alike): the K steps of its weight-gradient tiles.
__global__ void __launch_bounds__(1024) bwd_prepare_kernel(const int4* __restrict__ groups, int G,
                                                           int E, int* __restrict__ seg_off,
                                                           int2* __restrict__ segs,
                                                           const int32_t* __restrict__ err) {
  __shared__ int s_cnt[1025];
  __shared__ int s_scan[33];
  if (block_should_stop(err)) return;
  for (int e = threadIdx.x; e < E; e += blockDim.x) s_cnt[e] = 0;
  __syncthreads();
  for (int g = threadIdx.x; g < G; g += blockDim.x) {
    const int4 r = groups[g];
    if (r.y > 0) atomicAdd(&s_cnt[r.z], 1);
  }
  __syncthreads();
  const int nseg = block_exclusive_scan(s_cnt, E, s_scan);
  for (int e = threadIdx.x; e < E; e += blockDim.x) seg_off[e] = s_cnt[e];
  __syncthreads();  // thread 0 reuses s_cnt as its fill cursor below
  if (threadIdx.x == 0) {
    seg_off[E] = nseg;
    // stable fill in group-table order (one thread: at most 4096 records)
    for (int g = 0; g < G; ++g) {
      const int4 r = groups[g];
      if (r.y > 0) segs[s_cnt[r.z]++] = make_int2(r.x, r.y);
    }
  }
}

// Tiled transpose of 16-bit elements, 64 x 64 per block, 16-byte loads and stores:
// out[c][q] = in[q][c] for q < n_out.  cols, n_out and the row pitches are multiples of 8
// elements.  With f16_to_bf16 the fp16 inputs are rounded to bf16 on the way.  Batched over
// blockIdx.z.  (The backward uses it for W2 -> W2^T in bf16.)
constexpr int kTp = 64;
// shared tile [q][c]: the 16-byte chunk j of row q is stored at chunk j ^ ((q / 8) % 8), so
// that reading one column across rows q = 8i + r (i = 0..7) touches 8 different banks
__global__ void __launch_bounds__(256) transpose_kernel(
    const uint16_t* __restrict__ in, int cols, int64_t ld_in, int64_t in_bstride,
    uint16_t* __restrict__ out, int64_t ld_out, int64_t out_bstride, int n_out, int f16_to_bf16,
    const int32_t* __restrict__ err) {
  __shared__ __align__(16) uint16_t tile[kTp][kTp];
  if (load_err(err)) return;
  const int q0 = blockIdx.x * kTp, c0 = blockIdx.y * kTp;
  const int nq = n_out;
  if (q0 >= nq) return;
  const uint16_t* src = in + (int64_t)blockIdx.z * in_bstride;
  uint16_t* dst = out + (int64_t)blockIdx.z * out_bstride;
  for (int i = threadIdx.x; i < kTp * 8; i += blockDim.x) {
    const int q = i >> 3, ch = i & 7;
    const int c = c0 + ch * 8;
    const int r = q0 + q < nq ? q0 + q : -1;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (r >= 0 && c < cols) {
      v = __ldg(reinterpret_cast<const uint4*>(src + (int64_t)r * ld_in + c));
      if (f16_to_bf16) {
        uint32_t* w = reinterpret_cast<uint32_t*>(&v);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[j]));
          const __nv_bfloat162 bb = __floats2bfloat162_rn(f.x, f.y);
          w[j] = *reinterpret_cast<const uint32_t*>(&bb);
        }
      }
    }
    *reinterpret_cast<uint4*>(&tile[q][(ch ^ ((q >> 3) & 7)) * 8]) = v;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < kTp * 8; i += blockDim.x) {
    const int c = i >> 3, qc = i & 7;
    if (c0 + c >= cols || q0 + qc * 8 >= nq) continue;
    // rows qc*8 .. qc*8+7 share (q / 8) = qc: column c sits in chunk (c / 8) ^ qc
    const int col = (((c >> 3) ^ qc) << 3) | (c & 7);
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
      w[j] = (uint32_t)tile[qc * 8 + 2 * j][col] | ((uint32_t)tile[qc * 8 + 2 * j + 1][col] << 16);
    // n_out is a multiple of 8: whole 16-byte chunks
    *reinterpret_cast<uint4*>(dst + (int64_t)(c0 + c) * ld_out + q0 + qc * 8) =
        make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// Backward of combine: dy[perm[t,j]] = gate[t,j] * dout[t] (bf16), dgate[t,j] =
// <dout[t], y[perm[t,j]]> (fp32).  One warp per token, 16-byte vectors.
// YSrc / DySink (rows.cuh): y read and dy written on this GPU, or on every rank of the
// expert-parallel layer through its row tables (peer loads and stores).
// U: 16-byte vectors of each row per lane per step (8 for rows of d >= 4096: 847 -> 707 us at
// d = 7168; 4 below, where 8 gains nothing)
template <class YSrc, class DySink, int U>
__global__ void __launch_bounds__(256) combine_backward_kernel(
    const uint4* __restrict__ dout, const __grid_constant__ YSrc y, const int32_t* __restrict__ perm,
    const float* __restrict__ gate, int T, int k, int dv, const __grid_constant__ DySink dy,
    float* __restrict__ dgate, const int32_t* __restrict__ err) {
  if (load_err(err)) return;
  const int lane = threadIdx.x & 31;
  const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t t = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); t < T; t += nwarps) {
    for (int j = 0; j < k; ++j) {
      const int r = __ldg(perm + t * k + j);
      const float gj = __ldg(gate + t * k + j);
      const uint4* yr = y.row(r, dv);
      uint4* dyr = dy.row(r, dv);
      // U vectors of dout and of y in flight per lane before the first FMA; the partial
      // dot products are summed in a fixed order, so the result does not depend on timing
      float dot[U];
#pragma unroll
      for (int u = 0; u < U; ++u) dot[u] = 0.f;
      for (int v0 = lane; v0 < dv; v0 += 32 * U) {
        uint4 a[U], b[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int v = v0 + 32 * u;
          if (v < dv) {
            a[u] = __ldg(dout + t * dv + v);
            b[u] = __ldcs(yr + v);
          }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int v = v0 + 32 * u;
          if (v < dv) {
            const __nv_bfloat162* ap = reinterpret_cast<const __nv_bfloat162*>(&a[u]);
            const __nv_bfloat162* bp = reinterpret_cast<const __nv_bfloat162*>(&b[u]);
            uint32_t o[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const float2 af = __bfloat1622float2(ap[i]);
              const float2 bf = __bfloat1622float2(bp[i]);
              dot[u] = fmaf(af.x, bf.x, dot[u]);
              dot[u] = fmaf(af.y, bf.y, dot[u]);
              o[i] = pack_bf16(gj * af.x, gj * af.y);
            }
            dyr[v] = make_uint4(o[0], o[1], o[2], o[3]);
          }
        }
      }
      float total = 0.f;
#pragma unroll
      for (int u = 0; u < U; ++u) total += dot[u];
      total = warp_sum(total);
      if (lane == 0) dgate[t * k + j] = total;
    }
  }
}

// Backward of the gates (softmax over the chosen logits): dlogit[t, idx[t,j]] =
// gate[t,j] (dgate[t,j] - sum_i gate[t,i] dgate[t,i]); every other logit gets 0.
__global__ void __launch_bounds__(256) topk_backward_kernel(
    const float* __restrict__ gate, const float* __restrict__ dgate,
    const int32_t* __restrict__ idx, int T, int E, int k, float* __restrict__ dlogits,
    const int32_t* __restrict__ err) {
  if (load_err(err)) return;
  const int lane = threadIdx.x & 31;
  const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t t = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); t < T; t += nwarps) {
    const float g = lane < k ? __ldg(gate + t * k + lane) : 0.f;
    const float dg = lane < k ? __ldg(dgate + t * k + lane) : 0.f;
    const float s = warp_sum(g * dg);
    float* row = dlogits + t * E;
    for (int e = lane; e < E; e += 32) row[e] = 0.f;
    __syncwarp();
    if (lane < k) row[__ldg(idx + t * k + lane)] = g * (dg - s);
  }
}

// ------------------------------------------------------------------- host side
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn_bwd() {
  static EncodeTiledFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 2-D 16-bit tensor [rows, cols], row pitch `ld` elements, box 64 columns x box_rows rows,
// 128-byte swizzle.
bool make_map16(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int64_t ld,
                int box_rows, bool bf16) {
  EncodeTiledFn fn = encode_fn_bwd();
  if (!fn || rows <= 0 || cols <= 0) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
  cuuint32_t box[2] = {(cuuint32_t)BK, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2,
            const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

size_t bwd_smem_bytes() {
  return 1024 + (size_t)STAGES * STAGE_BYTES + 4 * 32 * 32 * 4 + (2 * STAGES + 5) * 8 + 4 * 4 +
         (MAX_GROUPS + 1) * 4 + 33 * 4;
}

// Output map of the weight-gradient tiles: fp32 [rows, cols] (row stride ld), 32 x 32
// boxes, the 128-byte swizzle of the staging blocks.
bool make_map_out32(CUtensorMap* m, void* base, int64_t rows, int64_t cols, int64_t ld) {
  EncodeTiledFn fn = encode_fn_bwd();
  if (!fn || rows <= 0 || cols <= 0) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)ld * 4};
  cuuint32_t box[2] = {32, 32};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, base, dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int EPI, bool WGRAD, bool BMN = false>
int launch_bwd_gemm(const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1,
                    const CUtensorMap& p0, const CUtensorMap& p1, const BwdArgs& args,
                    cudaStream_t s, const CUtensorMap* out = nullptr) {
  static bool configured[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  const size_t smem = bwd_smem_bytes();
  if (dev < 64 && !configured[dev]) {
    if (cudaFuncSetAttribute(bwd_gemm_kernel<EPI, WGRAD, BMN>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
      return MOE_ERR_LAUNCH;
    configured[dev] = true;
  }
  bwd_gemm_kernel<EPI, WGRAD, BMN><<<num_sms(), BWD_THREADS, smem, s>>>(a, b0, b1, p0, p1,
                                                                     out ? *out : a, args);
  return launch_status();
}

// out[c][q] = in[q][c] for q < n_out (see transpose_kernel), batched.
int transpose(const void* in, int cols, int64_t ld_in, int64_t in_bstride, void* out,
              int64_t ld_out, int64_t out_bstride, int n_out, int batches, bool f16_to_bf16,
              const int32_t* err,
              cudaStream_t s) {
  if (cols <= 0 || n_out <= 0 || batches <= 0) return MOE_OK;
  dim3 grid((n_out + kTp - 1) / kTp, (cols + kTp - 1) / kTp, batches);
  transpose_kernel<<<grid, 256, 0, s>>>(static_cast<const uint16_t*>(in), cols, ld_in, in_bstride,
                                        static_cast<uint16_t*>(out), ld_out, out_bstride, n_out,
                                        f16_to_bf16 ? 1 : 0, err);
  return launch_status();
}

// Workspace carve-up (every piece 256-byte aligned).  RC rows, Eo experts in the weight
// gradients (the home experts, then -- for a rank of the expert-parallel layer -- its pool
// slots), G group records.
struct BwdWs {
  __nv_bfloat16* w2t;   // [Eo*F, d] (W2, and the pool's P2, transposed, rounded to bf16)
  float* dh;            // [RC, F]
  __nv_bfloat16* dgu;   // [RC, 2F]
  __nv_bfloat16* hb;    // [RC, F] h = silu(g) u recomputed, bf16
  int* seg_off;         // [Eo+1]
  int2* segs;           // [G]
  int64_t bytes;
};

BwdWs carve(uint8_t* base, int64_t RC, int Eo, int d, int F, int G) {
  BwdWs w{};
  int64_t off = 0;
  auto take = [&](int64_t bytes) {
    const int64_t at = off;
    off += (bytes + 255) / 256 * 256;
    return base ? base + at : nullptr;
  };
  w.w2t = reinterpret_cast<__nv_bfloat16*>(take((int64_t)Eo * F * d * 2));
  w.dh = reinterpret_cast<float*>(take(RC * F * 4));
  w.dgu = reinterpret_cast<__nv_bfloat16*>(take(RC * 2 * F * 2));
  w.hb = reinterpret_cast<__nv_bfloat16*>(take(RC * F * 2));
  w.seg_off = reinterpret_cast<int*>(take((int64_t)(Eo + 1) * 4));
  w.segs = reinterpret_cast<int2*>(take((int64_t)G * 8));
  w.bytes = off;
  return w;
}

// The grouped-FFN backward over a group table of G records {row_start, rows, weight index,
// -} on RC rows: weight index z < e_home reads the home tensors (W1, W3, W2), z >= e_home
// pool slot z - e_home (P1, P3, P2, n_pool slots); the weight gradients dW* hold Eo =
// e_home + n_pool entries, each the sum over every group with that index.
int grouped_ffn_backward_impl(const __nv_bfloat16* recv, const __nv_bfloat16* dy,
                              const int4* groups, int G, int64_t RC, int e_home, int n_pool,
                              const __nv_bfloat16* W1, const __nv_bfloat16* W3, const __half* W2,
                              const __nv_bfloat16* P1, const __nv_bfloat16* P3, const __half* P2,
                              int d, int F, __nv_bfloat16* dx_rows, float* dW1, float* dW3,
                              float* dW2, void* workspace, int64_t workspace_bytes, int32_t* err,
                              cudaStream_t s) {
  const int Eo = e_home + n_pool;
  BwdWs w = carve(static_cast<uint8_t*>(workspace), RC, Eo, d, F, G);
  if (w.bytes > workspace_bytes) return MOE_ERR_ARG;
  int st;
  // weight gradients of entries without rows are zero; the GEMMs below write every tile
  // (an entry with no K steps stores zeros), and with no rows nothing else runs
  if (RC == 0) {
    if (cudaMemsetAsync(dW1, 0, (size_t)Eo * F * d * 4, s) != cudaSuccess ||
        cudaMemsetAsync(dW3, 0, (size_t)Eo * F * d * 4, s) != cudaSuccess ||
        cudaMemsetAsync(dW2, 0, (size_t)Eo * d * F * 4, s) != cudaSuccess)
      return MOE_ERR_LAUNCH;
    return MOE_OK;
  }
  // 1. per-entry lists of group row ranges (the weight gradients' K steps)
  bwd_prepare_kernel<<<1, 1024, 0, s>>>(groups, G, Eo, w.seg_off, w.segs, err);
  if ((st = launch_status()) != MOE_OK) return st;
  // 2. W2T[z] = W2[z]^T [F,d], rounded to bf16, the pool's slots after the home experts (the
  //    dH GEMM reads it K-major; W1 and W3 are read MN-major by the dX GEMM, no copy)
  if ((st = transpose(W2, F, F, (int64_t)d * F, w.w2t, d, (int64_t)F * d, d, e_home, true, err,
                      s)))
    return st;
  if (n_pool > 0 &&
      (st = transpose(P2, F, F, (int64_t)d * F, w.w2t + (int64_t)e_home * F * d, d,
                      (int64_t)F * d, d, n_pool, true, err, s)))
    return st;
  const int bnF = (F % 256 == 0) ? 256 : 128;
  const int bnD = (d % 256 == 0) ? 256 : 128;
  BwdArgs base{};
  base.groups = groups;
  base.G = G;
  base.err = err;
  base.E = Eo;
  base.F = F;
  base.e_home = Eo;  // dH reads W2T, which holds every entry
  // 3. dH = dY W2 (per group, fp32 out)
  {
    CUtensorMap ma, mb;
    if (!make_map16(&ma, dy, RC, d, d, BM, true) ||
        !make_map16(&mb, w.w2t, (int64_t)Eo * F, d, d, bnF, true))
      return MOE_ERR_DEVICE;
    BwdArgs a = base;
    a.n_blocks_n = F / bnF;
    a.k_blocks = d / BK;
    a.bn_out = bnF;
    a.mma_n = bnF;
    a.rows_per_expert = F;
    a.out_ld = F;
    a.bf16 = 1;
    a.out = w.dh;
    if ((st = launch_bwd_gemm<EPI_F32, false>(ma, mb, mb, mb, mb, a, s))) return st;
  }
  // 4. dG, dU: the gate/up GEMM re-run on the rows, SwiGLU backward in the epilogue (which
  //    also stores h = silu(g) u in bf16 for dW2)
  {
    CUtensorMap ma, m1, m3, p1, p3;
    if (!make_map16(&ma, recv, RC, d, d, BM, true) ||
        !make_map16(&m1, W1, (int64_t)e_home * F, d, d, 128, true) ||
        !make_map16(&m3, W3, (int64_t)e_home * F, d, d, 128, true))
      return MOE_ERR_DEVICE;
    if (n_pool > 0) {
      if (!make_map16(&p1, P1, (int64_t)n_pool * F, d, d, 128, true) ||
          !make_map16(&p3, P3, (int64_t)n_pool * F, d, d, 128, true))
        return MOE_ERR_DEVICE;
    } else {
      p1 = m1;
      p3 = m3;
    }
    BwdArgs a = base;
    a.e_home = e_home;
    a.n_blocks_n = F / 128;
    a.k_blocks = d / BK;
    a.bn_out = 128;
    a.mma_n = 256;
    a.rows_per_expert = F;
    a.out_ld = 2 * F;
    a.bf16 = 1;
    a.dh = w.dh;
    a.dgu = w.dgu;
    a.hb = w.hb;
    if ((st = launch_bwd_gemm<EPI_SWIGLU_BWD, false>(ma, m1, m3, p1, p3, a, s))) return st;
  }
  // 5. dX rows = [dG | dU] [W1; W3] (K = 2F, bf16): B read MN-major from W1 (K steps below
  //    F/64) and W3 (the rest), each as [rows, d columns] in boxes of 64 x 64
  {
    CUtensorMap ma, m1, m3, p1, p3;
    if (!make_map16(&ma, w.dgu, RC, 2 * F, 2 * F, BM, true) ||
        !make_map16(&m1, W1, (int64_t)e_home * F, d, d, 64, true) ||
        !make_map16(&m3, W3, (int64_t)e_home * F, d, d, 64, true))
      return MOE_ERR_DEVICE;
    if (n_pool > 0) {
      if (!make_map16(&p1, P1, (int64_t)n_pool * F, d, d, 64, true) ||
          !make_map16(&p3, P3, (int64_t)n_pool * F, d, d, 64, true))
        return MOE_ERR_DEVICE;
    } else {
      p1 = m1;
      p3 = m3;
    }
    BwdArgs a = base;
    a.e_home = e_home;
    a.n_blocks_n = d / bnD;
    a.k_blocks = 2 * F / BK;
    a.kb_split = F / BK;
    a.bn_out = bnD;
    a.mma_n = bnD;
    a.rows_per_expert = F;
    a.out_ld = d;
    a.bf16 = 1;
    a.out = dx_rows;
    if ((st = launch_bwd_gemm<EPI_BF16, false, true>(ma, m1, m3, p1, p3, a, s))) return st;
  }
  // 6. weight gradients, every group of an entry in one accumulator (on one GPU: a home
  //    expert's home and replica groups alike); A and B are the row-major activations
  //    read MN-major in boxes of 64 rows x 64 columns
  {
    CUtensorMap ma, mb;
    if (!make_map16(&ma, dy, RC, d, d, 64, true) || !make_map16(&mb, w.hb, RC, F, F, 64, true))
      return MOE_ERR_DEVICE;
    BwdArgs a = base;
    a.n_blocks_n = F / bnF;
    a.bn_out = bnF;
    a.mma_n = bnF;
    a.out_ld = F;
    a.bf16 = 1;
    a.out = dW2;
    a.seg_off = w.seg_off;
    a.segs = w.segs;
    a.m_blocks = d / BM;
    a.a_row_base = 0;
    a.out_expert_stride = (int64_t)d * F;
    CUtensorMap mo;
    if (!make_map_out32(&mo, dW2, (int64_t)Eo * d, F, F)) return MOE_ERR_DEVICE;
    if ((st = launch_bwd_gemm<EPI_F32, true>(ma, mb, mb, mb, mb, a, s, &mo))) return st;
  }
  {
    CUtensorMap ma, mb;
    if (!make_map16(&ma, w.dgu, RC, 2 * F, 2 * F, 64, true) ||
        !make_map16(&mb, recv, RC, d, d, 64, true))
      return MOE_ERR_DEVICE;
    BwdArgs a = base;
    a.n_blocks_n = d / bnD;
    a.bn_out = bnD;
    a.mma_n = bnD;
    a.out_ld = d;
    a.bf16 = 1;
    a.seg_off = w.seg_off;
    a.segs = w.segs;
    a.m_blocks = F / BM;
    a.out_expert_stride = (int64_t)F * d;
    a.a_row_base = 0;
    a.out = dW1;
    CUtensorMap mo1, mo3;
    if (!make_map_out32(&mo1, dW1, (int64_t)Eo * F, d, d) ||
        !make_map_out32(&mo3, dW3, (int64_t)Eo * F, d, d))
      return MOE_ERR_DEVICE;
    if ((st = launch_bwd_gemm<EPI_F32, true>(ma, mb, mb, mb, mb, a, s, &mo1))) return st;
    a.a_row_base = F;
    a.out = dW3;
    if ((st = launch_bwd_gemm<EPI_F32, true>(ma, mb, mb, mb, mb, a, s, &mo3))) return st;
  }
  return MOE_OK;
}

// Replica gradients reduced back home across ranks, in place: home expert e_local of rank me
// (entry e_local of its own partials) gets, in (rank, slot) order, the partial of every pool
// slot (v, s) of the job's plan that held a copy of it, read from rank v's partials through
// the rank tables; an expert without copies is left as it is.  parts[p][v] -> rank v's
// [B+S][n4] partials of projection p (fp32, 16-byte vectors).
struct RankParts {
  const float4* p[3][MOE_EP_MAX_RANKS];
};

__global__ void __launch_bounds__(256) ep_reduce_home_kernel(
    const int32_t* __restrict__ rep, int W, int me, int B, int S, int64_t n4,
    const __grid_constant__ RankParts parts, const int32_t* __restrict__ err) {
  __shared__ int s_src[MOE_EP_MAX_RANKS];  // v * S + s of the copies, in order (a rank's
                                          // slots hold distinct experts: at most W copies)
  __shared__ int s_n;
  if (block_should_stop(err)) return;
  constexpr int kChunk = 256 * 4;  // float4 vectors per block and step
  const int64_t chunks = (n4 + kChunk - 1) / kChunk;
  const int64_t total = (int64_t)B * 3 * chunks;
  int cur = -1;
  for (int64_t w = blockIdx.x; w < total; w += gridDim.x) {
    const int el = (int)(w / (3 * chunks));
    const int64_t rem = w - (int64_t)el * 3 * chunks;
    const int proj = (int)(rem / chunks);
    const int64_t c = rem - (int64_t)proj * chunks;
    if (el != cur) {  // the copies of expert me*B + el, found once per expert
      __syncthreads();
      if (threadIdx.x == 0) {
        int n = 0;
        const int e = me * B + el;
        for (int q = 0; q < W * S && n < MOE_EP_MAX_RANKS; ++q)
          if (__ldg(rep + q) == e) s_src[n++] = q;
        s_n = n;
      }
      __syncthreads();
      cur = el;
    }
    const int n = s_n;
    if (n == 0) continue;
    float4* own = const_cast<float4*>(parts.p[proj][me]) + (int64_t)el * n4;
    for (int64_t v = c * kChunk + threadIdx.x; v < min(n4, (c + 1) * kChunk); v += blockDim.x) {
      float4 a = own[v];
      for (int i = 0; i < n; ++i) {
        const int q = s_src[i];
        const float4 b = __ldcs(parts.p[proj][q / S] + (int64_t)(B + q % S) * n4 + v);
        a.x += b.x;
        a.y += b.y;
        a.z += b.z;
        a.w += b.w;
      }
      own[v] = a;
    }
  }
}

}  // namespace

int64_t ffn_backward_workspace_bytes(int T, int k, int E, int R, int S, int d, int F, int G) {
  (void)R;
  (void)S;
  return carve(nullptr, (int64_t)T * k, E, d, F, G).bytes;
}

int64_t ep_ffn_backward_workspace_bytes(int T, int k, int E, int W, int S, int d, int F) {
  const int B = E / W;
  return carve(nullptr, (int64_t)T * k, B + S, d, F, B + S).bytes;
}

int launch_combine_backward(const __nv_bfloat16* dout, const __nv_bfloat16* y,
                            const int32_t* perm, const float* gate, int T, int k, int d,
                            __nv_bfloat16* dy, float* dgate, const int32_t* err,
                            cudaStream_t s) {
  if (T == 0) return MOE_OK;
  const int64_t want = ((int64_t)T + 7) / 8;
  const int64_t cap = (int64_t)num_sms() * 8;
  const unsigned grid = (unsigned)(want < cap ? want : cap);
  const LocalY yv{reinterpret_cast<const uint4*>(y)};
  const LocalRows dv{reinterpret_cast<uint4*>(dy)};
  if (d / 8 >= 512)
    combine_backward_kernel<LocalY, LocalRows, 8><<<grid, 256, 0, s>>>(
        reinterpret_cast<const uint4*>(dout), yv, perm, gate, T, k, d / 8, dv, dgate, err);
  else
    combine_backward_kernel<LocalY, LocalRows, 4><<<grid, 256, 0, s>>>(
        reinterpret_cast<const uint4*>(dout), yv, perm, gate, T, k, d / 8, dv, dgate, err);
  return launch_status();
}

int launch_topk_backward(const float* gate, const float* dgate, const int32_t* idx, int T, int E,
                         int k, float* dlogits, const int32_t* err, cudaStream_t s) {
  if (T == 0) return MOE_OK;
  const int64_t want = ((int64_t)T + 7) / 8;
  const int64_t cap = (int64_t)num_sms() * 8;
  topk_backward_kernel<<<(unsigned)(want < cap ? want : cap), 256, 0, s>>>(gate, dgate, idx, T, E,
                                                                           k, dlogits, err);
  return launch_status();
}

int launch_grouped_ffn_backward(const __nv_bfloat16* recv, const __nv_bfloat16* dy,
                                const __half* h,
                                const int32_t* plan, const moe_plan_layout& L,
                                const __nv_bfloat16* W1, const __nv_bfloat16* W3,
                                const __half* W2, int T, int k, int E, int R, int S, int d,
                                int F, __nv_bfloat16* dx_rows, float* dW1, float* dW3,
                                float* dW2, void* workspace, int64_t workspace_bytes,
                                int32_t* err, cudaStream_t s) {
  (void)h;  // not read: the SwiGLU-backward epilogue recomputes h (in bf16) for dW2
  (void)S;
  // the plan's groups name their expert in z; every group reads the home tensors
  return grouped_ffn_backward_impl(recv, dy, reinterpret_cast<const int4*>(plan + L.groups),
                                   R * L.max_groups_per_rank, (int64_t)T * k, E, 0, W1, W3, W2,
                                   nullptr, nullptr, nullptr, d, F, dx_rows, dW1, dW3, dW2,
                                   workspace, workspace_bytes, err, s);
}

int launch_ep_combine_backward(const __nv_bfloat16* dout, const __nv_bfloat16* const* y_ranks,
                               const int32_t* perm, const float* gate, int W, int T, int k, int d,
                               __nv_bfloat16* const* dy_ranks, float* dgate, const int32_t* err,
                               cudaStream_t s) {
  if (T == 0) return MOE_OK;
  RankY yv;
  RankRows dv;
  for (int u = 0; u < MOE_EP_MAX_RANKS; ++u) {
    yv.base[u] = u < W ? reinterpret_cast<const uint4*>(y_ranks[u]) : nullptr;
    dv.base[u] = u < W ? reinterpret_cast<uint4*>(dy_ranks[u]) : nullptr;
  }
  yv.C = dv.C = T * k;
  const int64_t want = ((int64_t)T + 7) / 8;
  const int64_t cap = (int64_t)num_sms() * 8;
  const unsigned grid = (unsigned)(want < cap ? want : cap);
  if (d / 8 >= 512)  // as the single-GPU launcher, so both sum in the same order
    combine_backward_kernel<RankY, RankRows, 8><<<grid, 256, 0, s>>>(
        reinterpret_cast<const uint4*>(dout), yv, perm, gate, T, k, d / 8, dv, dgate, err);
  else
    combine_backward_kernel<RankY, RankRows, 4><<<grid, 256, 0, s>>>(
        reinterpret_cast<const uint4*>(dout), yv, perm, gate, T, k, d / 8, dv, dgate, err);
  return launch_status();
}

int launch_ep_grouped_ffn_backward(const __nv_bfloat16* recv, const __nv_bfloat16* dy,
                                   const int32_t* groups, int B, int S, int C,
                                   const __nv_bfloat16* W1, const __nv_bfloat16* W3,
                                   const __half* W2, const __nv_bfloat16* P1,
                                   const __nv_bfloat16* P3, const __half* P2, int d, int F,
                                   __nv_bfloat16* dx_rows, float* dP1, float* dP3, float* dP2,
                                   void* workspace, int64_t workspace_bytes, int32_t* err,
                                   cudaStream_t s) {
  // the re-based group table names each group's weights in z: home expert 0..B-1, pool
  // slot B + s
  return grouped_ffn_backward_impl(recv, dy, reinterpret_cast<const int4*>(groups), B + S,
                                   (int64_t)C, B, S, W1, W3, W2, P1, P3, P2, d, F, dx_rows, dP1,
                                   dP3, dP2, workspace, workspace_bytes, err, s);
}

int launch_ep_reduce_home(const int32_t* plan, const moe_plan_layout& L,
                          float* const* part1_ranks, float* const* part3_ranks,
                          float* const* part2_ranks, int W, int me, int E, int S, int d, int F,
                          const int32_t* err, cudaStream_t s) {
  RankParts parts;
  for (int u = 0; u < MOE_EP_MAX_RANKS; ++u) {
    parts.p[0][u] = u < W ? reinterpret_cast<const float4*>(part1_ranks[u]) : nullptr;
    parts.p[1][u] = u < W ? reinterpret_cast<const float4*>(part3_ranks[u]) : nullptr;
    parts.p[2][u] = u < W ? reinterpret_cast<const float4*>(part2_ranks[u]) : nullptr;
  }
  const int64_t n4 = (int64_t)d * F / 4;
  ep_reduce_home_kernel<<<num_sms() * 4, 256, 0, s>>>(plan + L.replica_expert, W, me, E / W, S,
                                                     n4, parts, err);
  return launch_status();
}

}  // namespace moe
