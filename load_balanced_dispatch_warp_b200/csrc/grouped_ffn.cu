// Grouped SwiGLU expert FFN on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// "DeepEP-on-EFA Guidance, section 1: What is MoE", phase (c): each rank runs its local
// experts over the rows it received as a batched grouped GEMM.  Here the ranks' rows are
// one buffer [R*C, d] and the plan's group table names, for each contiguous run of rows,
// the expert (home tensor) or the pool slot (replica) whose weights it uses.
//
//   GEMM 1:  h = silu(X W1^T) * (X W3^T)   per group; one MMA of N = 2*128 covers a
//            128-column block of W1 and the same block of W3, so the SwiGLU epilogue
//            reads gate and up values of the same row from one TMEM accumulator.
//   GEMM 2:  y = h W2^T                    per group; N = 256 (128 when d % 256 != 0).
//            h and W2 are fp16: rounding h to bf16 (8-bit significand) would put the
//            worst element of y near the 1e-2 parity bound at F/d >= 2, fp16's 11 bits
//            keep it below half of it at the same tensor-core rate.
//
// Kernel shape (one CTA per SM, persistent, 192 threads):
//   warp 0      TMA producer: A (128 rows x 64 K) and B (N rows x 64 K) tiles, 128-byte
//               swizzle, into a 4-stage ring; mbarrier transaction counts signal arrival.
//   warp 1      TMEM owner (alloc/dealloc of 512 columns) and single-thread MMA issuer:
//               tcgen05.mma.cta_group::1.kind::f16, bf16 x bf16 -> fp32 in TMEM, two
//               accumulator buffers of 256 columns so the epilogue of one tile overlaps
//               the main loop of the next.
//   warps 2-5   epilogue: tcgen05.ld 32 lanes x 32 columns at a time, SwiGLU or plain
//               conversion to bf16, masked row stores (a tile's rows past the end of its
//               group belong to the next group and are not written).
// Tiles are (group, 128-row block, N block), enumerated m-block-major from a prefix over
// the group table built in shared memory by every CTA; CTA i takes tiles i, i+grid, ...
//
// Gathered GEMM 1 (GATHER): row r of the A operand is the token row x[src[r]] instead of
// a dispatched copy recv[r] -- the dispatch's row copy folded into the operand load, as
// the zero-copy dispatch of the MoonEP news article (paragraph 3) and the fused kernels of
// "DeepEP-on-EFA Guidance, section 1: What is MoE" (routing layout and data movement in
// dedicated GPU kernels) describe.  The whole producer warp then writes
// each A tile with 16-byte cp.async copies into the same 128-byte-swizzled layout TMA
// produces (16-byte chunk c of tile row r at r*128 + ((c ^ (r % 8)) * 16)); one warp
// instruction reads four whole 128-byte row segments.  Rows past the group's end are
// zero-filled.  After its copies for a stage each lane posts an arrival that fires when
// they have landed (cp.async.mbarrier.arrive.noinc), so the producer never blocks on
// them; the stage's full barrier expects those 32 arrivals plus the B operand's
// transaction bytes.
//
// Every mbarrier wait is bounded (about 2 s of %globaltimer); a wait that runs out sets
// MOE_DERR_TIMEOUT and a shared abort flag, every role leaves its loop, the producer
// waits (bounded) for its copies in flight, the MMA thread for its MMAs, and TMEM is
// freed before the CTA exits.
#include <cuda.h>

#include <atomic>

#include "common.cuh"

namespace moe {
namespace {

constexpr int BM = 128;          // rows per tile (TMEM lanes)
constexpr int BK = 64;           // K per stage: 64 bf16 = one 128-byte swizzle row
constexpr int UMMA_K = 16;       // K per tcgen05.mma for 16-bit inputs
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;        // 16 KiB
constexpr int B_BYTES_MAX = 256 * BK * 2;   // 32 KiB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES_MAX;
constexpr int ACC_COLS = 256;               // one accumulator buffer
constexpr int TMEM_COLS = 2 * ACC_COLS;
constexpr int MAX_GROUPS = 4096;
constexpr int FFN_THREADS = 192;
constexpr uint64_t WAIT_LIMIT_NS = 2000000000ull;

struct FfnArgs {
  const int4* groups;   // [G] {row_start, rows, expert, weight_ref}, rows == -1 unused
  int G;
  int uniform_rows;     // > 0: no table; group g = {g*uniform_rows, uniform_rows, g, g}
  int half_tiles;       // 1: a tile with at most 64 valid rows runs M = 64 MMAs
  int n_chunk;          // > 0: a group's tiles run chunk by chunk of n_chunk weight
                        //    blocks, every row block of the group within a chunk (1:
                        //    weight-block-major); 0: row-block-major
  int n_blocks_n;       // output column blocks per row block
  int k_blocks;         // K / BK
  int bn_out;           // output columns per tile (128 for SwiGLU, N for plain)
  int mma_n;            // N of the MMA (256 for SwiGLU, bn_out for plain)
  int rows_per_expert;  // rows of one expert in the B tensors: F (GEMM 1) or d (GEMM 2)
  int E;
  int out_ld;           // columns of the output tensor
  void* out;            // h (fp16) for GEMM 1, y (bf16) for GEMM 2
  int32_t* err;
  const __nv_bfloat16* gx;  // GATHER: token rows x [T, gd]
  const int32_t* gsrc;      // GATHER: token of each row, [R*C]
  int gd;                   // GATHER: row length of x (= d)
  int gT;                   // GATHER: rows of x (tokens)
  // fused combine (GEMM 2 only, when comb_out != nullptr): the epilogue adds
  // gate[t,j] * y_row into comb_out[t] (fp32 [T, out_ld]) for the token t = comb_src[row]
  // and the choice j with comb_perm[t,j] == row, instead of storing y
  float* comb_out;
  const int32_t* comb_src;
  const int32_t* comb_perm;
  const float* comb_gate;
  int comb_k;
};

// --------------------------------------------------------------------- PTX wrappers
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

// Bounded wait for the phase of `parity` to complete.  Returns false (and raises the
// abort flag and the error bit) if the bound runs out, or if another role aborted.
__device__ __noinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                       int32_t* err, uint64_t limit_ns = WAIT_LIMIT_NS) {
  if (mbar_try(bar, parity)) return true;
  uint64_t t0 = 0;
  for (uint32_t it = 1;; ++it) {
    if (mbar_try(bar, parity)) return true;
    if ((it & 255u) == 0) {
      if (*abort_flag) return false;
      const uint64_t now = globaltimer();
      if (t0 == 0) {
        t0 = now;
      } else if (now - t0 > limit_ns) {
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

// 16-byte global -> shared copy, bytes past src_bytes (0 or 16) zero-filled, L2 only
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(src_bytes)
               : "memory");
}
// arrival on `bar` once every cp.async this thread issued so far has landed (counts as one
// of the barrier's expected arrivals)
__device__ __forceinline__ void cp_async_arrive(uint32_t bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_all;" ::: "memory");
}
// make this thread's completed shared-memory writes visible to the async proxy (MMA)
__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
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
// 32 TMEM lanes x 32 consecutive 32-bit columns: thread i of the warp gets lane base+i.
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

// Shared-memory matrix descriptor of a K-major tile written by TMA with the 128-byte
// swizzle: rows of 128 bytes, 8-row atoms 1024 bytes apart (stride byte offset), leading
// byte offset unused for swizzled K-major (encoded 1), descriptor version 1 (bits 46-47),
// layout type 2 = 128-byte swizzle (bits 61-63).  Stepping K by 16 elements inside the
// 128-byte row adds 32 bytes to the start address.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)1 << 16) |
         ((uint64_t)(1024 >> 4) << 32) | ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}
// Instruction descriptor, kind::f16: fp32 accumulate (bits 4-5 = 1), A and B of one type,
// bf16 (1) or fp16 (0), at bits 7-9 and 10-12, both K-major (bits 15, 16 = 0), N >> 3 at
// bits 17-22, M >> 4 at bits 24-28.
__host__ __device__ constexpr uint32_t make_idesc(int M, int N, bool bf16) {
  return (1u << 4) | ((bf16 ? 1u : 0u) << 7) | ((bf16 ? 1u : 0u) << 10) |
         ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}
// fp16 pair with saturation to +-65504 (no infinities from large activations)
__device__ __forceinline__ uint32_t pack_f16_sat(float a, float b) {
  a = fminf(fmaxf(a, -65504.0f), 65504.0f);
  b = fminf(fmaxf(b, -65504.0f), 65504.0f);
  __half2 v = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ float silu(float z) { return z / (1.0f + __expf(-z)); }

// Group g: from the plan's table, or (fixed-capacity layout) expert g's block of
// uniform_rows rows with its home weights.
__device__ __forceinline__ int4 group_of(const FfnArgs& a, int g) {
  if (a.uniform_rows > 0) return make_int4(g * a.uniform_rows, a.uniform_rows, g, g);
  return __ldg(a.groups + g);
}

struct Tile {
  int a_row;       // first row of the A block
  int valid_rows;  // rows of the block inside the group (<= BM)
  bool half;       // M = 64 tile: 64-row A box, M = 64 MMAs, accumulator rows 16 per lane
                   // quadrant (row r in TMEM lane 32 (r / 16) + r % 16, measured)
  int b_row;       // first row of the B block inside its tensor
  bool pool;       // B from the replica pool instead of the home tensors
  int n_block;
};

__device__ __forceinline__ Tile decode_tile(int t, const FfnArgs& a, const int* s_prefix) {
  const int mt = t / a.n_blocks_n;
  Tile tl;
  tl.n_block = t - mt * a.n_blocks_n;
  // last group whose prefix <= mt (empty groups share their successor's prefix)
  int lo = 0, hi = a.G - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (s_prefix[mid] <= mt) lo = mid; else hi = mid - 1;
  }
  const int4 g = group_of(a, lo);
  int m_local = mt - s_prefix[lo];
  if (a.n_chunk > 0) {
    const int local = t - s_prefix[lo] * a.n_blocks_n;
    const int mc = s_prefix[lo + 1] - s_prefix[lo];
    const int per_chunk = mc * a.n_chunk;
    const int c = local / per_chunk;
    const int rem = local - c * per_chunk;
    const int ncw = min(a.n_chunk, a.n_blocks_n - c * a.n_chunk);  // the last chunk may be narrower
    m_local = rem / ncw;
    tl.n_block = c * a.n_chunk + (rem - m_local * ncw);
  }
  tl.a_row = g.x + m_local * BM;
  tl.valid_rows = min(BM, g.y - m_local * BM);
  tl.half = a.half_tiles && tl.valid_rows <= BM / 2;
  const int ref = g.w;
  tl.pool = ref >= a.E;
  tl.b_row = (tl.pool ? ref - a.E : ref) * a.rows_per_expert + tl.n_block * a.bn_out;
  return tl;
}

template <bool SWIGLU, bool GATHER>
__global__ void __launch_bounds__(FFN_THREADS, 1)
    ffn_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_a64,
               const __grid_constant__ CUtensorMap tm_b0, const __grid_constant__ CUtensorMap tm_b1,
               const __grid_constant__ CUtensorMap tm_p0, const __grid_constant__ CUtensorMap tm_p1,
               const FfnArgs args) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte alignment for the swizzle atoms
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* stage_base = smem;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
  // bars: full[STAGES], empty[STAGES], tfull[2], tempty[2], drain
  int* s_misc = reinterpret_cast<int*>(bars + 2 * STAGES + 5);  // [0] tmem base, [1] abort, [2] err0
  int* s_prefix = s_misc + 4;                                     // [G + 1]
  int* s_scan = s_prefix + MAX_GROUPS + 1;                        // 33 ints

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  volatile int* abort_flag = s_misc + 1;

  if (tid == 0) {
    s_misc[2] = load_err(args.err);
    s_misc[1] = 0;
  }
  __syncthreads();
  if (s_misc[2] != 0) return;

  // m-blocks per group, exclusive prefix over the group table
  for (int g = tid; g < args.G; g += blockDim.x) {
    const int rows = group_of(args, g).y;
    s_prefix[g] = rows > 0 ? (rows + BM - 1) / BM : 0;
  }
  __syncthreads();
  const int total_m = block_exclusive_scan(s_prefix, args.G, s_scan);
  if (tid == 0) s_prefix[args.G] = total_m;
  const int total_tiles = total_m * args.n_blocks_n;

  const uint32_t full0 = smem_u32(bars);
  const uint32_t empty0 = smem_u32(bars + STAGES);
  const uint32_t tfull0 = smem_u32(bars + 2 * STAGES);
  const uint32_t tempty0 = smem_u32(bars + 2 * STAGES + 2);
  const uint32_t drain = smem_u32(bars + 2 * STAGES + 4);
  if (tid == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full0 + 8 * s, GATHER ? 33 : 1);
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

  if (warp == 0 && GATHER) {
    // ------------------------------------------------ gathering producer (whole warp)
    const int q = lane >> 3;             // row within each 4-row slice
    const int c = lane & 7;              // 16-byte chunk of the 128-byte row segment
    const char* xb = reinterpret_cast<const char*>(args.gx) + c * 16;
    const int64_t row_bytes = (int64_t)args.gd * 2;
    int stage = 0;
    uint32_t phase = 0;
    uint32_t issued_mask = 0, issued_phase = 0;
    bool ok = true;
    for (int t = blockIdx.x; ok && t < total_tiles; t += gridDim.x) {
      const Tile tl = decode_tile(t, args, s_prefix);
      // tokens of rows lane + 32 m; copy i covers row 4 i + q
      int tokv[4];
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const int r = lane + 32 * m;
        int tv = r < tl.valid_rows ? __ldg(args.gsrc + tl.a_row + r) : 0;
        if ((unsigned)tv >= (unsigned)args.gT) {  // never read outside x
          atomicOr(args.err, MOE_DERR_ID_RANGE);
          tv = 0;
        }
        tokv[m] = tv;
      }
      int tok[32];
      uint32_t vmask = 0;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const int r = 4 * i + q;
        tok[i] = __shfl_sync(MOE_FULL_MASK, tokv[i >> 3], r & 31);
        vmask |= (r < tl.valid_rows ? 1u : 0u) << i;
      }
      for (int kb = 0; kb < args.k_blocks; ++kb) {
        // every lane waits (bounded); the warp goes on only if all of them saw the stage free
        if (!__all_sync(MOE_FULL_MASK, mbar_wait(empty0 + 8 * stage, phase ^ 1u, abort_flag, args.err))) {
          ok = false;
          break;
        }
        const uint32_t fb = full0 + 8 * stage;
        const uint32_t sa = smem_u32(stage_base + stage * STAGE_BYTES);
        const char* kbase = xb + (int64_t)kb * (BK * 2);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int r = 4 * i + q;
          const int rs = r & 7;
          const uint32_t dst = sa + ((uint32_t)(r >> 3) << 10) + ((uint32_t)rs << 7) +
                               ((uint32_t)(c ^ rs) << 4);
          cp_async16(dst, kbase + (int64_t)tok[i] * row_bytes, ((vmask >> i) & 1u) * 16u);
        }
        cp_async_arrive(fb);
        if (lane == 0) {
          const CUtensorMap* mb0 = tl.pool ? &tm_p0 : &tm_b0;
          const CUtensorMap* mb1 = tl.pool ? &tm_p1 : &tm_b1;
          const uint32_t sb = sa + A_BYTES;
          mbar_expect_tx(fb, b_bytes);
          tma_load_2d(sb, mb0, fb, kb * BK, tl.b_row);
          tma_load_2d(sb + (b_bytes >> 1), mb1, fb, kb * BK, tl.b_row);
        }
        issued_mask |= 1u << stage;
        issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      }
    }
    // no copy of this warp may still be landing when the CTA leaves
    cp_async_wait_all();
    __syncwarp();
    if (lane == 0) {
      for (int s = 0; s < STAGES; ++s)
        if (issued_mask & (1u << s)) {
          volatile int no_abort = 0;
          mbar_wait(full0 + 8 * s, (issued_phase >> s) & 1u, &no_abort, args.err);
        }
    }
    __syncwarp();
  } else if (warp == 0) {
    // ------------------------------------------------------------- TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0, issued_phase = 0;  // per stage: issued at least once, parity
      for (int t = blockIdx.x; t < total_tiles; t += gridDim.x) {
        const Tile tl = decode_tile(t, args, s_prefix);
        const CUtensorMap* mb0 = tl.pool ? &tm_p0 : &tm_b0;
        const CUtensorMap* mb1 = tl.pool ? &tm_p1 : &tm_b1;
        bool ok = true;
        for (int kb = 0; kb < args.k_blocks; ++kb) {
          if (!mbar_wait(empty0 + 8 * stage, phase ^ 1u, abort_flag, args.err)) { ok = false; break; }
          const uint32_t fb = full0 + 8 * stage;
          const uint32_t sa = smem_u32(stage_base + stage * STAGE_BYTES);
          const uint32_t sb = sa + A_BYTES;
          mbar_expect_tx(fb, (tl.half ? A_BYTES / 2 : A_BYTES) + b_bytes);
          tma_load_2d(sa, tl.half ? &tm_a64 : &tm_a, fb, kb * BK, tl.a_row);
          if (SWIGLU) {
            tma_load_2d(sb, mb0, fb, kb * BK, tl.b_row);
            tma_load_2d(sb + (b_bytes >> 1), mb1, fb, kb * BK, tl.b_row);
          } else {
            tma_load_2d(sb, mb0, fb, kb * BK, tl.b_row);
          }
          issued_mask |= 1u << stage;
          issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
      }
      // make sure no copy is still landing in shared memory when the CTA leaves
      for (int s = 0; s < STAGES; ++s)
        if (issued_mask & (1u << s)) {
          volatile int no_abort = 0;
          mbar_wait(full0 + 8 * s, (issued_phase >> s) & 1u, &no_abort, args.err);
        }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      // GEMM 1: x, W1, W3 in bf16; GEMM 2: h and W2 in fp16
      const uint32_t idesc_full = make_idesc(BM, args.mma_n, SWIGLU);
      const uint32_t idesc_half = make_idesc(BM / 2, args.mma_n, SWIGLU);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      for (int t = blockIdx.x; t < total_tiles; t += gridDim.x) {
        const uint32_t idesc = decode_tile(t, args, s_prefix).half ? idesc_half : idesc_full;
        if (!mbar_wait(tempty0 + 8 * acc, acc_phase ^ 1u, abort_flag, args.err)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * ACC_COLS;
        bool ok = true;
        for (int kb = 0; kb < args.k_blocks; ++kb) {
          if (!mbar_wait(full0 + 8 * stage, phase, abort_flag, args.err)) { ok = false; break; }
          if (GATHER) fence_proxy_async();  // A written by cp.async (generic proxy)
          tc_fence_after();
          const uint32_t sa = smem_u32(stage_base + stage * STAGE_BYTES);
          const uint32_t sb = sa + A_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / UMMA_K; ++kk)
            tc_mma(d_tmem, sw128_desc(sa + kk * UMMA_K * 2), sw128_desc(sb + kk * UMMA_K * 2), idesc,
                   (kb | kk) != 0);
          tc_commit(empty0 + 8 * stage);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        tc_commit(tfull0 + 8 * acc);
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      }
      // all MMAs issued by this thread have completed once `drain` flips
      tc_commit(drain);
      volatile int no_abort = 0;
      mbar_wait(drain, 0, &no_abort, args.err);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------- epilogue (warps 2-5)
    const int quarter = warp & 3;  // TMEM lanes this warp may access
    const int r_in = quarter * 32 + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = blockIdx.x; t < total_tiles; t += gridDim.x) {
      const Tile tl = decode_tile(t, args, s_prefix);
      const bool ok = mbar_wait(tfull0 + 8 * acc, acc_phase, abort_flag, args.err);
      if (!__all_sync(MOE_FULL_MASK, ok)) break;  // warp-uniform exit
      tc_fence_after();
      const uint32_t tbase = tmem_base + ((uint32_t)(quarter * 32) << 16) + acc * ACC_COLS;
      // an M = 64 tile holds its row 16 q + i in lane i < 16 of quadrant q
      const int row = tl.half ? quarter * 16 + lane : r_in;
      const bool valid = (!tl.half || lane < 16) && row < tl.valid_rows;
      // both outputs are 16-bit: h (fp16) after GEMM 1, y (bf16) after GEMM 2
      uint16_t* orow = static_cast<uint16_t*>(args.out) + (int64_t)(tl.a_row + row) * args.out_ld +
                       (int64_t)tl.n_block * args.bn_out;
      if (SWIGLU) {
#pragma unroll 1
        for (int c = 0; c < 128 / 32; ++c) {
          uint32_t g[32], u[32];
          tmem_ld32(tbase + c * 32, g);
          tmem_ld32(tbase + 128 + c * 32, u);
          tmem_wait_ld();
          uint32_t p[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float g0 = __uint_as_float(g[2 * i]), g1 = __uint_as_float(g[2 * i + 1]);
            const float u0 = __uint_as_float(u[2 * i]), u1 = __uint_as_float(u[2 * i + 1]);
            p[i] = pack_f16_sat(silu(g0) * u0, silu(g1) * u1);
          }
          if (valid) {
            uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
            for (int i = 0; i < 4; ++i) dst[i] = make_uint4(p[4 * i], p[4 * i + 1], p[4 * i + 2], p[4 * i + 3]);
          }
        }
      } else if (args.comb_out != nullptr) {
        // fused combine: this row's token and gate, then gate * y added into the token's
        // fp32 output row (16-byte vector atomics, performed at L2)
        int64_t tok = 0;
        float gsc = 0.f;
        bool live = valid;
        if (live) {
          const int r = tl.a_row + row;
          tok = __ldg(args.comb_src + r);
          if (tok < 0 || tok >= args.gT) {  // never touch a row outside the output
            atomicOr(args.err, MOE_DERR_ID_RANGE);
            live = false;
            tok = 0;
          } else {
            for (int j = 0; j < args.comb_k; ++j)
              if (__ldg(args.comb_perm + tok * args.comb_k + j) == r)
                gsc = __ldg(args.comb_gate + tok * args.comb_k + j);
          }
        }
        float* crow = args.comb_out + tok * args.out_ld + (int64_t)tl.n_block * args.bn_out;
#pragma unroll 1
        for (int c = 0; c < args.bn_out / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(tbase + c * 32, v);
          tmem_wait_ld();
          if (live) {
#pragma unroll
            for (int i = 0; i < 8; ++i)
              atomicAdd(reinterpret_cast<float4*>(crow + c * 32 + 4 * i),
                        make_float4(gsc * __uint_as_float(v[4 * i]), gsc * __uint_as_float(v[4 * i + 1]),
                                    gsc * __uint_as_float(v[4 * i + 2]), gsc * __uint_as_float(v[4 * i + 3])));
          }
        }
      } else {
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

// ----------------------------------------------------------------- CTA-pair variant
//
// The same two GEMMs with the 2-SM tensor-core instruction (tcgen05.mma.cta_group::2):
// two CTAs of a cluster compute one 256-row x N tile.  CTA v of the pair holds rows
// [128 v, 128 v + 128) of A and columns [v N/2, (v+1) N/2) of B in its own shared memory
// and receives the accumulator of its 128 rows (all N columns) in its own TMEM; the
// tensor cores of the two SMs exchange the B halves.  Each SM therefore loads 16 KiB of A
// and N/2 * 128 bytes of B per K step instead of 16 KiB + N * 128 bytes: a third fewer
// operand bytes per MAC at N = 256, at the price of 256-row padding of each group's last
// tile.  For GEMM 1, CTA 0's B half is the W1 block and CTA 1's the W3 block, so the
// accumulator columns are still gate | up and the SwiGLU epilogue is unchanged.
//
// Protocol (leader = CTA rank 0):
//   full[s]    leader only: the leader's producer posts the transaction bytes of both
//              CTAs' copies; both CTAs' TMA copies (.cta_group::2) complete on it.
//   empty[s]   in both CTAs: one commit of the leader's MMA thread arrives on both.
//   tfull[b]   in both CTAs: the same, after a tile's K loop.
//   tempty[b]  leader only: 8 arrivals, one per epilogue warp of either CTA.
//   drain      in both CTAs: committed after the last MMA, before TMEM is freed.
// TMEM (512 columns, two accumulators of 256) is allocated and freed by warp 1 of both
// CTAs with cta_group::2.  Barrier initialisation is published to the peer by a cluster
// barrier before any role starts, and neither CTA leaves before a cluster barrier that
// follows the last access to the other's shared memory.  A stale error word read by one
// CTA of a pair and not the other cannot split the pair: the two CTAs OR their reads.
constexpr int P_STAGES = 6;
constexpr int P_BM = 2 * BM;                  // rows per pair tile
constexpr int P_B_BYTES_MAX = 128 * BK * 2;   // this CTA's half of B at N = 256
constexpr int P_STAGE_BYTES = A_BYTES + P_B_BYTES_MAX;

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_id_x() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_count_x() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
  return r;
}
// shared::cluster address of the variable at shared::cta address `saddr` in CTA `rank`
__device__ __forceinline__ uint32_t map_to_rank(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}
__device__ __forceinline__ uint32_t ld_cluster_u32(uint32_t caddr) {
  uint32_t v;
  asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(caddr) : "memory");
  return v;
}
// every thread of both CTAs
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\t"
               "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_remote(uint32_t caddr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(caddr)
               : "memory");
}
// TMA copy into this CTA's shared memory whose completion is counted on `bar_c`, a
// shared::cluster barrier address that may lie in the peer CTA
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map,
                                                 uint32_t bar_c, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar_c)
      : "memory");
}
// Arrival, once every pair MMA issued so far has completed, on the barrier at shared
// offset `bar` in both CTAs of the pair (CTA mask 0b11).  A commit, not a copy: nothing is
// loaded through the cluster.
__device__ __forceinline__ void tc_commit_pair(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(bar),
      "h"((uint16_t)3)
      : "memory");
}
__device__ __forceinline__ void tc_mma_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// This CTA's part of pair tile t: its 128 rows and its half of the B columns.  A group's
// last block with at most 128 rows left is a half tile (with half_tiles and N = 256): an
// M = 128 pair MMA, 64 rows in each CTA.
__device__ __forceinline__ Tile decode_pair_tile(int t, const FfnArgs& a, const int* s_prefix,
                                                 int rank, bool swiglu) {
  const int mt = t / a.n_blocks_n;
  Tile tl;
  tl.n_block = t - mt * a.n_blocks_n;
  int lo = 0, hi = a.G - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (s_prefix[mid] <= mt) lo = mid; else hi = mid - 1;
  }
  const int4 g = group_of(a, lo);
  int m_local = mt - s_prefix[lo];
  if (a.n_chunk > 0) {  // the group's weight blocks chunk by chunk, as decode_tile
    const int local = t - s_prefix[lo] * a.n_blocks_n;
    const int mc = s_prefix[lo + 1] - s_prefix[lo];
    const int per_chunk = mc * a.n_chunk;
    const int c = local / per_chunk;
    const int rem = local - c * per_chunk;
    const int ncw = min(a.n_chunk, a.n_blocks_n - c * a.n_chunk);
    m_local = rem / ncw;
    tl.n_block = c * a.n_chunk + (rem - m_local * ncw);
  }
  const int base = m_local * P_BM;  // first row of the pair tile in the group
  tl.half = a.half_tiles && a.mma_n == 256 && g.y - base <= BM;
  const int rows_cta = tl.half ? BM / 2 : BM;
  const int first = base + rank * rows_cta;  // this CTA's first row inside the group
  tl.a_row = g.x + first;
  tl.valid_rows = max(0, min(rows_cta, g.y - first));
  const int ref = g.w;
  tl.pool = ref >= a.E;
  tl.b_row = (tl.pool ? ref - a.E : ref) * a.rows_per_expert + tl.n_block * a.bn_out +
             (swiglu ? 0 : rank * (a.mma_n >> 1));
  return tl;
}

template <bool SWIGLU>
__global__ void __launch_bounds__(FFN_THREADS, 1)
    ffn_pair_kernel(const __grid_constant__ CUtensorMap tm_a,
                    const __grid_constant__ CUtensorMap tm_a64,
                    const __grid_constant__ CUtensorMap tm_b0,
                    const __grid_constant__ CUtensorMap tm_b1,
                    const __grid_constant__ CUtensorMap tm_p0,
                    const __grid_constant__ CUtensorMap tm_p1, const FfnArgs args) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* stage_base = smem;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + P_STAGES * P_STAGE_BYTES);
  // bars: full[P_STAGES], empty[P_STAGES], tfull[2], tempty[2], drain
  int* s_misc = reinterpret_cast<int*>(bars + 2 * P_STAGES + 5);
  // s_misc: [0] tmem base, [1] abort, [2] error word seen by this CTA, [3] by the pair
  int* s_prefix = s_misc + 4;
  int* s_scan = s_prefix + MAX_GROUPS + 1;
  // half tiles of GEMM 1: the up warps hand their values to the gate warps through
  // s_xchg ([2][32 rows][32 floats]) under the barriers xfull (up written) and xempty
  // (read)
  uint64_t* xbars = reinterpret_cast<uint64_t*>((reinterpret_cast<uintptr_t>(s_scan + 33) + 7) &
                                                ~static_cast<uintptr_t>(7));
  float* s_xchg = reinterpret_cast<float*>((reinterpret_cast<uintptr_t>(xbars + 2) + 15) &
                                           ~static_cast<uintptr_t>(15));

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  volatile int* abort_flag = s_misc + 1;

  const uint32_t full0 = smem_u32(bars);
  const uint32_t empty0 = smem_u32(bars + P_STAGES);
  const uint32_t tfull0 = smem_u32(bars + 2 * P_STAGES);
  const uint32_t tempty0 = smem_u32(bars + 2 * P_STAGES + 2);
  const uint32_t drain = smem_u32(bars + 2 * P_STAGES + 4);
  if (tid == 0) {
    s_misc[1] = 0;
    s_misc[2] = load_err(args.err);
    for (int s = 0; s < P_STAGES; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(tfull0 + 8 * b, 1);
      mbar_init(tempty0 + 8 * b, 8);
    }
    mbar_init(drain, 1);
    mbar_init(smem_u32(xbars), 2);      // xfull: the two up warps
    mbar_init(smem_u32(xbars + 1), 2);  // xempty: the two gate warps
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  for (int g = tid; g < args.G; g += blockDim.x) {
    const int rows = group_of(args, g).y;
    s_prefix[g] = rows > 0 ? (rows + P_BM - 1) / P_BM : 0;
  }
  __syncthreads();
  const int total_m = block_exclusive_scan(s_prefix, args.G, s_scan);
  if (tid == 0) s_prefix[args.G] = total_m;
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(s_misc)),
                 "r"(TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  cluster_sync_all();  // barriers initialised and TMEM allocated in both CTAs
  tc_fence_after();
  if (tid == 0) s_misc[3] = s_misc[2] | (int)ld_cluster_u32(map_to_rank(smem_u32(s_misc + 2), rank ^ 1u));
  __syncthreads();
  const int total_tiles = s_misc[3] != 0 ? 0 : total_m * args.n_blocks_n;
  const uint32_t tmem_base = static_cast<uint32_t>(s_misc[0]);
  const int first_tile = (int)cluster_id_x();
  const int tile_step = (int)cluster_count_x();

  if (warp == 0) {
    // ------------------------------------------------------------- TMA producer
    if (lane == 0) {
      const uint32_t b_half = (uint32_t)(args.mma_n >> 1) * BK * 2;
      const uint32_t tx = 2u * (A_BYTES + b_half);
      const uint32_t tx_half = 2u * (A_BYTES / 2 + b_half);  // 64-row A boxes
      const uint32_t full_leader0 = map_to_rank(full0, 0);
      const CUtensorMap* home = (SWIGLU && rank == 1) ? &tm_b1 : &tm_b0;
      const CUtensorMap* pool = (SWIGLU && rank == 1) ? &tm_p1 : &tm_p0;
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0, issued_phase = 0;
      bool ok = true;
      for (int t = first_tile; ok && t < total_tiles; t += tile_step) {
        const Tile tl = decode_pair_tile(t, args, s_prefix, (int)rank, SWIGLU);
        const CUtensorMap* mb = tl.pool ? pool : home;
        for (int kb = 0; kb < args.k_blocks; ++kb) {
          if (!mbar_wait(empty0 + 8 * stage, phase ^ 1u, abort_flag, args.err)) { ok = false; break; }
          const uint32_t sa = smem_u32(stage_base + stage * P_STAGE_BYTES);
          if (leader) mbar_expect_tx(full0 + 8 * stage, tl.half ? tx_half : tx);
          tma_load_2d_pair(sa, tl.half ? &tm_a64 : &tm_a, full_leader0 + 8 * stage, kb * BK,
                           tl.a_row);
          tma_load_2d_pair(sa + A_BYTES, mb, full_leader0 + 8 * stage, kb * BK, tl.b_row);
          issued_mask |= 1u << stage;
          issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
          if (++stage == P_STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      // No copy may still be landing when either CTA leaves.  The leader's full barriers
      // count both CTAs' bytes; the peer sees its stages consumed on its empty barriers.
      for (int s = 0; s < P_STAGES; ++s)
        if (issued_mask & (1u << s)) {
          volatile int no_abort = 0;
          const uint32_t par = (issued_phase >> s) & 1u;
          if (leader) {
            mbar_wait(full0 + 8 * s, par, &no_abort, args.err);
          } else if (!mbar_wait(empty0 + 8 * s, par, ok ? &no_abort : abort_flag, args.err)) {
            const uint64_t t0 = globaltimer();  // error path: let copies in flight land
            while (globaltimer() - t0 < 100000ull) {
            }
          }
        }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer (leader CTA only)
    if (lane == 0 && leader) {
      const uint32_t idesc_full = make_idesc(P_BM, args.mma_n, SWIGLU);
      const uint32_t idesc_half = make_idesc(BM, args.mma_n, SWIGLU);  // 64 rows per CTA
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      for (int t = first_tile; t < total_tiles; t += tile_step) {
        const uint32_t idesc =
            decode_pair_tile(t, args, s_prefix, 0, SWIGLU).half ? idesc_half : idesc_full;
        if (!mbar_wait(tempty0 + 8 * acc, acc_phase ^ 1u, abort_flag, args.err)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * ACC_COLS;
        bool ok = true;
        for (int kb = 0; kb < args.k_blocks; ++kb) {
          if (!mbar_wait(full0 + 8 * stage, phase, abort_flag, args.err)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = smem_u32(stage_base + stage * P_STAGE_BYTES);
          const uint32_t sb = sa + A_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / UMMA_K; ++kk)
            tc_mma_pair(d_tmem, sw128_desc(sa + kk * UMMA_K * 2), sw128_desc(sb + kk * UMMA_K * 2),
                        idesc, (kb | kk) != 0);
          tc_commit_pair(empty0 + 8 * stage);
          if (++stage == P_STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        tc_commit_pair(tfull0 + 8 * acc);
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      }
      tc_commit_pair(drain);
    }
    if (lane == 0) {
      // both CTAs: every MMA that reads this CTA's shared memory or writes its TMEM is done
      volatile int no_abort = 0;
      mbar_wait(drain, 0, &no_abort, args.err);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------ epilogue (warps 2-5)
    // Full tiles: lane = row (this CTA's 128), columns as N.  Half tiles (M = 128 pair
    // MMA, measured layout): this CTA's 64 rows sit in lanes 0-63 with output columns
    // 0-127 and again in lanes 64-127 with columns 128-255, both in TMEM columns 0-127.
    // In GEMM 1 the first half is gate and the second up: the up warps (quarters 2, 3)
    // pass their values to the gate warps (quarters 0, 1) of the same rows through shared
    // memory.
    const int quarter = warp & 3;
    const int r_in = quarter * 32 + lane;
    const uint32_t tempty_leader0 = map_to_rank(tempty0, 0);
    const uint32_t xfull = smem_u32(xbars), xempty = smem_u32(xbars + 1);
    uint32_t xphase = 0;
    bool xok = true;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = first_tile; xok && t < total_tiles; t += tile_step) {
      const Tile tl = decode_pair_tile(t, args, s_prefix, (int)rank, SWIGLU);
      const bool ok = mbar_wait(tfull0 + 8 * acc, acc_phase, abort_flag, args.err);
      if (!__all_sync(MOE_FULL_MASK, ok)) break;
      tc_fence_after();
      const uint32_t tbase = tmem_base + ((uint32_t)(quarter * 32) << 16) + acc * ACC_COLS;
      if (tl.half) {
        const int hrow = (quarter & 1) * 32 + lane;  // row among this CTA's 64
        const bool hvalid = hrow < tl.valid_rows;
        float* stg = s_xchg + (quarter & 1) * 1024;  // [32 rows][32 floats]
        if (SWIGLU) {
          uint16_t* orow = static_cast<uint16_t*>(args.out) +
                           (int64_t)(tl.a_row + hrow) * args.out_ld +
                           (int64_t)tl.n_block * args.bn_out;
#pragma unroll 1
          for (int c = 0; c < 128 / 32; ++c) {
            uint32_t v[32];
            tmem_ld32(tbase + c * 32, v);
            tmem_wait_ld();
            if (quarter >= 2) {
              // up: wait until the gate warps have read the previous chunk, then stage
              // row `lane`'s 32 values (16-byte chunk j at j ^ (lane % 8): no conflicts)
              const bool w = mbar_wait(xempty, xphase ^ 1u, abort_flag, args.err);
              if (!__all_sync(MOE_FULL_MASK, w)) { xok = false; break; }
#pragma unroll
              for (int j = 0; j < 8; ++j)
                *reinterpret_cast<uint4*>(stg + lane * 32 + ((j ^ (lane & 7)) << 2)) =
                    make_uint4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
              __syncwarp();
              if (lane == 0) mbar_arrive(xfull);
            } else {
              const bool w = mbar_wait(xfull, xphase, abort_flag, args.err);
              if (!__all_sync(MOE_FULL_MASK, w)) { xok = false; break; }
              uint32_t u[32];
#pragma unroll
              for (int j = 0; j < 8; ++j) {
                const uint4 q = *reinterpret_cast<const uint4*>(stg + lane * 32 + ((j ^ (lane & 7)) << 2));
                u[4 * j] = q.x;
                u[4 * j + 1] = q.y;
                u[4 * j + 2] = q.z;
                u[4 * j + 3] = q.w;
              }
              __syncwarp();
              if (lane == 0) mbar_arrive(xempty);
              uint32_t p[16];
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                const float g0 = __uint_as_float(v[2 * i]), g1 = __uint_as_float(v[2 * i + 1]);
                const float u0 = __uint_as_float(u[2 * i]), u1 = __uint_as_float(u[2 * i + 1]);
                p[i] = pack_f16_sat(silu(g0) * u0, silu(g1) * u1);
              }
              if (hvalid) {
                uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
                for (int i = 0; i < 4; ++i) dst[i] = make_uint4(p[4 * i], p[4 * i + 1], p[4 * i + 2], p[4 * i + 3]);
              }
            }
            xphase ^= 1u;
          }
        } else {
          uint16_t* orow = static_cast<uint16_t*>(args.out) +
                           (int64_t)(tl.a_row + hrow) * args.out_ld +
                           (int64_t)tl.n_block * args.bn_out + (quarter >> 1) * 128;
#pragma unroll 1
          for (int c = 0; c < 128 / 32; ++c) {
            uint32_t v[32];
            tmem_ld32(tbase + c * 32, v);
            tmem_wait_ld();
            uint32_t p[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) p[i] = pack_bf16(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
            if (hvalid) {
              uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
              for (int i = 0; i < 4; ++i) dst[i] = make_uint4(p[4 * i], p[4 * i + 1], p[4 * i + 2], p[4 * i + 3]);
            }
          }
        }
      } else {
      const bool valid = r_in < tl.valid_rows;
      uint16_t* orow = static_cast<uint16_t*>(args.out) + (int64_t)(tl.a_row + r_in) * args.out_ld +
                       (int64_t)tl.n_block * args.bn_out;
      if (SWIGLU) {
#pragma unroll 1
        for (int c = 0; c < 128 / 32; ++c) {
          uint32_t g[32], u[32];
          tmem_ld32(tbase + c * 32, g);
          tmem_ld32(tbase + 128 + c * 32, u);
          tmem_wait_ld();
          uint32_t p[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float g0 = __uint_as_float(g[2 * i]), g1 = __uint_as_float(g[2 * i + 1]);
            const float u0 = __uint_as_float(u[2 * i]), u1 = __uint_as_float(u[2 * i + 1]);
            p[i] = pack_f16_sat(silu(g0) * u0, silu(g1) * u1);
          }
          if (valid) {
            uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
            for (int i = 0; i < 4; ++i) dst[i] = make_uint4(p[4 * i], p[4 * i + 1], p[4 * i + 2], p[4 * i + 3]);
          }
        }
      } else {
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
      }
      if (!xok) break;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(tempty_leader0 + 8 * acc);
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
  }

  tc_fence_before();
  cluster_sync_all();  // all roles of both CTAs done
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(TMEM_COLS)
                 : "memory");
  }
  cluster_sync_all();
}

// Self-test of the bounded wait: one thread waits on an mbarrier that nothing arrives at,
// with a short limit; the wait gives up, sets MOE_DERR_TIMEOUT and the kernel returns.
__global__ void bounded_wait_selftest_kernel(int32_t* err, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(smem_u32(&bar), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    mbar_wait(smem_u32(&bar), 0, &abort_flag, err, limit_ns);
  }
}

// ----------------------------------------------------------------------------- host side
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
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

// 2-D 16-bit tensor [rows, cols] row-major, box = 64 columns x box_rows rows, 128-byte
// swizzle.
bool make_map(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int box_rows,
              CUtensorMapDataType type = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || rows <= 0) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  cuuint32_t box[2] = {(cuuint32_t)BK, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, type, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

size_t ffn_smem_bytes() {
  return 1024 + (size_t)STAGES * STAGE_BYTES + (2 * STAGES + 5) * 8 + 4 * 4 +
         (MAX_GROUPS + 1) * 4 + 33 * 4;
}

template <bool SWIGLU, bool GATHER>
int launch_one(const CUtensorMap& a, const CUtensorMap& a64, const CUtensorMap& b0,
               const CUtensorMap& b1, const CUtensorMap& p0, const CUtensorMap& p1,
               const FfnArgs& args, cudaStream_t s) {
  static bool configured[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  const size_t smem = ffn_smem_bytes();
  if (dev < 64 && !configured[dev]) {
    if (cudaFuncSetAttribute(ffn_kernel<SWIGLU, GATHER>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
      return MOE_ERR_LAUNCH;
    configured[dev] = true;
  }
  ffn_kernel<SWIGLU, GATHER><<<num_sms(), FFN_THREADS, smem, s>>>(a, a64, b0, b1, p0, p1, args);
  return launch_status();
}


size_t ffn_pair_smem_bytes() {
  return 1024 + (size_t)P_STAGES * P_STAGE_BYTES + (2 * P_STAGES + 5) * 8 + 4 * 4 +
         (MAX_GROUPS + 1) * 4 + 33 * 4 + 8 + 2 * 8 + 16 + 2 * 32 * 32 * 4;
}

std::atomic<int> g_ffn_tile_mode{0};  // 0: one CTA per 128-row tile, 1: CTA pairs
int g_pair_clusters[64] = {0};  // co-resident 2-CTA clusters per device

// Grid of the pair kernels: as many 2-CTA clusters as fit on the device at once (queried
// once per device; a GPC with an odd number of free SMs leaves one of them idle).
template <bool SWIGLU>
int launch_pair(const CUtensorMap& a, const CUtensorMap& a64, const CUtensorMap& b0,
                const CUtensorMap& b1, const CUtensorMap& p0, const CUtensorMap& p1,
                const FfnArgs& args, cudaStream_t s) {
  static bool configured[64] = {false};
  static int clusters[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 64) return MOE_ERR_LAUNCH;
  const size_t smem = ffn_pair_smem_bytes();
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(FFN_THREADS, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (!configured[dev]) {
    if (cudaFuncSetAttribute(ffn_pair_kernel<SWIGLU>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
      return MOE_ERR_LAUNCH;
    cfg.gridDim = dim3(2 * (num_sms() / 2), 1, 1);
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, ffn_pair_kernel<SWIGLU>, &cfg) != cudaSuccess || n <= 0) {
      cudaGetLastError();
      return MOE_ERR_LAUNCH;
    }
    clusters[dev] = n < num_sms() / 2 ? n : num_sms() / 2;
    g_pair_clusters[dev] = clusters[dev];
    configured[dev] = true;
  }
  cfg.gridDim = dim3(2 * clusters[dev], 1, 1);
  if (cudaLaunchKernelEx(&cfg, ffn_pair_kernel<SWIGLU>, a, a64, b0, b1, p0, p1, args) != cudaSuccess)
    return MOE_ERR_LAUNCH;
  return launch_status();
}

}  // namespace

int launch_bounded_wait_selftest(int32_t* err, int limit_us, cudaStream_t s) {
  bounded_wait_selftest_kernel<<<1, 32, 0, s>>>(err, (uint64_t)limit_us * 1000ull);
  return launch_status();
}

int set_ffn_tile_mode(int mode) {
  if (mode != 0 && mode != 1) return MOE_ERR_ARG;
  g_ffn_tile_mode.store(mode, std::memory_order_relaxed);
  return MOE_OK;
}

int ffn_tile_mode() { return g_ffn_tile_mode.load(std::memory_order_relaxed); }

int ffn_pair_clusters() {
  int dev = 0;
  cudaGetDevice(&dev);
  return dev < 64 ? g_pair_clusters[dev] : 0;
}

// Fused combine operands (moe_grouped_ffn_combine).
struct CombineArgs {
  float* out32;  // [T, d] fp32 accumulator, zeroed by the launcher
  const int32_t* src;
  const int32_t* perm;
  const float* gate;
  int k;
};

// out[i] = bf16(acc[i]), 8 values per thread and step (16-byte stores)
__global__ void __launch_bounds__(256) fp32_to_bf16_kernel(const float4* __restrict__ acc,
                                                           uint4* __restrict__ out, int64_t n8,
                                                           const int32_t* __restrict__ err) {
  if (load_err(err)) return;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n8;
       i += (int64_t)gridDim.x * blockDim.x) {
    const float4 a = __ldcs(acc + 2 * i), b = __ldcs(acc + 2 * i + 1);
    out[i] = make_uint4(pack_bf16(a.x, a.y), pack_bf16(a.z, a.w), pack_bf16(b.x, b.y),
                        pack_bf16(b.z, b.w));
  }
}

// GEMM 1 reads its rows from recv (x == nullptr) or gathers them as x[src[row]].  The
// groups come from `groups` (G entries) or, with uniform_rows > 0, are E blocks of
// uniform_rows rows; `rows` is the length of recv, h and y.
int launch_grouped_ffn_impl(const __nv_bfloat16* recv, const __nv_bfloat16* x,
                            const int32_t* src, const int4* groups, int G, int uniform_rows,
                            int64_t rows, const __nv_bfloat16* W1, const __nv_bfloat16* W3,
                            const __half* W2, const __nv_bfloat16* P1, const __nv_bfloat16* P3,
                            const __half* P2, int T, int E, int R, int S, int d, int F,
                            __half* h, __nv_bfloat16* y, int32_t* err, cudaStream_t s,
                            const CombineArgs* comb = nullptr) {
  if (rows == 0) return MOE_OK;
  const bool gather = x != nullptr;
  const bool pair = !gather && comb == nullptr &&
                    g_ffn_tile_mode.load(std::memory_order_relaxed) == 1;
  const int bn2 = (d % 256 == 0) ? 256 : 128;
  const int w2_box = pair ? bn2 / 2 : bn2;  // a pair CTA loads half of GEMM 2's B rows
  CUtensorMap m_recv, m_recv64, m_w1, m_w3, m_p1, m_p3, m_h, m_h64, m_w2, m_p2;
  if (!make_map(&m_w1, W1, (int64_t)E * F, d, 128) ||
      (!gather && !make_map(&m_recv, recv, rows, d, BM)) ||
      (!gather && !make_map(&m_recv64, recv, rows, d, BM / 2)) ||
      !make_map(&m_w3, W3, (int64_t)E * F, d, 128) ||
      !make_map(&m_h, h, rows, F, BM, CU_TENSOR_MAP_DATA_TYPE_FLOAT16) ||
      !make_map(&m_h64, h, rows, F, BM / 2, CU_TENSOR_MAP_DATA_TYPE_FLOAT16) ||
      !make_map(&m_w2, W2, (int64_t)E * d, F, w2_box, CU_TENSOR_MAP_DATA_TYPE_FLOAT16))
    return MOE_ERR_DEVICE;
  if (S > 0) {
    if (!make_map(&m_p1, P1, (int64_t)R * S * F, d, 128) ||
        !make_map(&m_p3, P3, (int64_t)R * S * F, d, 128) ||
        !make_map(&m_p2, P2, (int64_t)R * S * d, F, w2_box, CU_TENSOR_MAP_DATA_TYPE_FLOAT16))
      return MOE_ERR_DEVICE;
  } else {  // no pool: replica references cannot occur; pass the home maps
    m_p1 = m_w1;
    m_p3 = m_w3;
    m_p2 = m_w2;
  }
  FfnArgs a1;
  a1.groups = groups;
  a1.G = G;
  a1.uniform_rows = uniform_rows;
  a1.half_tiles = gather ? 0 : 1;  // the gathering producer always fills 128 rows
  a1.n_chunk = 2;  // measured fastest at the DeepSeek shape among 1, 2, 4 and row-block-major
  a1.comb_out = nullptr;
  a1.comb_src = nullptr;
  a1.comb_perm = nullptr;
  a1.comb_gate = nullptr;
  a1.comb_k = 0;
  a1.n_blocks_n = F / 128;
  a1.k_blocks = d / BK;
  a1.bn_out = 128;
  a1.mma_n = 256;
  a1.rows_per_expert = F;
  a1.E = E;
  a1.out_ld = F;
  a1.out = h;
  a1.err = err;
  a1.gx = x;
  a1.gsrc = src;
  a1.gd = d;
  a1.gT = T;
  int st = gather ? launch_one<true, true>(m_w1, m_w1, m_w1, m_w3, m_p1, m_p3, a1, s)
           : pair ? launch_pair<true>(m_recv, m_recv64, m_w1, m_w3, m_p1, m_p3, a1, s)
                  : launch_one<true, false>(m_recv, m_recv64, m_w1, m_w3, m_p1, m_p3, a1, s);
  if (st != MOE_OK) return st;
  FfnArgs a2 = a1;
  a2.n_blocks_n = d / bn2;
  a2.k_blocks = F / BK;
  a2.bn_out = bn2;
  a2.mma_n = bn2;
  a2.rows_per_expert = d;
  a2.out_ld = d;
  a2.out = y;
  a2.gx = nullptr;
  a2.gsrc = nullptr;
  a2.half_tiles = 1;
  if (comb != nullptr) {
    a2.comb_out = comb->out32;
    a2.comb_src = comb->src;
    a2.comb_perm = comb->perm;
    a2.comb_gate = comb->gate;
    a2.comb_k = comb->k;
  }
  return pair ? launch_pair<false>(m_h, m_h64, m_w2, m_w2, m_p2, m_p2, a2, s)
              : launch_one<false, false>(m_h, m_h64, m_w2, m_w2, m_p2, m_p2, a2, s);
}

int launch_grouped_ffn(const __nv_bfloat16* recv, const int32_t* plan,
                       const moe_plan_layout& L, const __nv_bfloat16* W1,
                       const __nv_bfloat16* W3, const __half* W2, const __nv_bfloat16* P1,
                       const __nv_bfloat16* P3, const __half* P2, int T, int k, int E, int R,
                       int S, int d, int F, __half* h, __nv_bfloat16* y, int32_t* err,
                       cudaStream_t s) {
  return launch_grouped_ffn_impl(recv, nullptr, nullptr,
                                 reinterpret_cast<const int4*>(plan + L.groups),
                                 R * L.max_groups_per_rank, 0, (int64_t)T * k, W1, W3, W2, P1,
                                 P3, P2, T, E, R, S, d, F, h, y, err, s);
}

int launch_grouped_ffn_gather(const __nv_bfloat16* x, const int32_t* src, const int32_t* plan,
                              const moe_plan_layout& L, const __nv_bfloat16* W1,
                              const __nv_bfloat16* W3, const __half* W2,
                              const __nv_bfloat16* P1, const __nv_bfloat16* P3,
                              const __half* P2, int T, int k, int E, int R, int S, int d, int F,
                              __half* h, __nv_bfloat16* y, int32_t* err, cudaStream_t s) {
  return launch_grouped_ffn_impl(nullptr, x, src, reinterpret_cast<const int4*>(plan + L.groups),
                                 R * L.max_groups_per_rank, 0, (int64_t)T * k, W1, W3, W2, P1,
                                 P3, P2, T, E, R, S, d, F, h, y, err, s);
}

int launch_grouped_ffn_combine(const __nv_bfloat16* recv, const int32_t* plan,
                               const moe_plan_layout& L, const __nv_bfloat16* W1,
                               const __nv_bfloat16* W3, const __half* W2,
                               const __nv_bfloat16* P1, const __nv_bfloat16* P3,
                               const __half* P2, const int32_t* src, const int32_t* perm,
                               const float* gate, int T, int k, int E, int R, int S, int d,
                               int F, __half* h, float* out32, __nv_bfloat16* out, int32_t* err,
                               cudaStream_t s) {
  if (T == 0) return MOE_OK;
  if (cudaMemsetAsync(out32, 0, sizeof(float) * (size_t)T * d, s) != cudaSuccess)
    return MOE_ERR_LAUNCH;
  CombineArgs comb{out32, src, perm, gate, k};
  const int st = launch_grouped_ffn_impl(recv, nullptr, nullptr,
                                         reinterpret_cast<const int4*>(plan + L.groups),
                                         R * L.max_groups_per_rank, 0, (int64_t)T * k, W1, W3,
                                         W2, P1, P3, P2, T, E, R, S, d, F, h, nullptr, err, s,
                                         &comb);
  if (st != MOE_OK) return st;
  const int64_t n8 = (int64_t)T * d / 8;
  const int64_t want = (n8 + 255) / 256;
  const int grid = (int)(want < (int64_t)num_sms() * 8 ? want : (int64_t)num_sms() * 8);
  fp32_to_bf16_kernel<<<grid, 256, 0, s>>>(reinterpret_cast<const float4*>(out32),
                                           reinterpret_cast<uint4*>(out), n8, err);
  return launch_status();
}

int launch_grouped_ffn_capacity(const __nv_bfloat16* recv, const __nv_bfloat16* W1,
                                const __nv_bfloat16* W3, const __half* W2, int E, int cap,
                                int d, int F, __half* h, __nv_bfloat16* y, int32_t* err,
                                cudaStream_t s) {
  if (cap == 0) return MOE_OK;
  return launch_grouped_ffn_impl(recv, nullptr, nullptr, nullptr, E, cap, (int64_t)E * cap, W1,
                                 W3, W2, nullptr, nullptr, nullptr, 0, E, 1, 0, d, F, h, y, err,
                                 s);
}

int launch_grouped_ffn_groups(const __nv_bfloat16* recv, const int32_t* groups, int G,
                              int64_t rows, const __nv_bfloat16* W1, const __nv_bfloat16* W3,
                              const __half* W2, const __nv_bfloat16* P1, const __nv_bfloat16* P3,
                              const __half* P2, int E, int S, int d, int F, __half* h,
                              __nv_bfloat16* y, int32_t* err, cudaStream_t s) {
  return launch_grouped_ffn_impl(recv, nullptr, nullptr, reinterpret_cast<const int4*>(groups), G,
                                 0, rows, W1, W3, W2, P1, P3, P2, 0, E, 1, S, d, F, h, y, err, s);
}

}  // namespace moe
