// tcgen05 flash attention for sm_100a (bf16 in, fp32 accumulate, head_dim 128).
//
// One kernel serves the three attention calls of the AReA hot path:
//   * coarse attention (Phase I: full-resolution queries against pooled keys),
//   * full attention (the operation AReA replaces, used for the speedup ratio),
//   * windowed attention (Phase II: queries of a window against its Halo
//     rectangle plus its global-KV tokens, outputs blended by tent weights).
// Pages: ai.info "Methodology in Plain English" (Phase I, Phase II);
// gpt-diffusion.com "Las dos fases de AReA".
//
// Design (one persistent CTA per SM; 320 threads for dense calls, 384 for
// window calls, whose warps 2-3 are idle and whose softmax warps are 4-11):
//   warp 0      producer: claims work units (window mode: from a counter in
//               the workspace, in the plan's parity-class order; dense mode:
//               statically), publishes one record per unit in a shared-memory
//               ring read by the other roles, and issues the TMA loads: Q
//               tiles once per unit, then a ring of K and V tiles (128 keys x
//               128 dims, 128B-swizzled, 32 KB each).  Dense rows use tiled
//               2-D loads.  Window keys are the global-KV list first (whole
//               tiles from the workspace's staging copy by one tiled load,
//               else rows copied with 16-byte cp.async by the 32 producer
//               lanes), then the Halo rectangle: 16x8-token patches (one 3-D
//               tiled box each) and 4x4-token cells on the strips the
//               patches leave (8 cells per tile, loaded by 8 lanes); window
//               queries come in 4x4 cells when the window's sides are
//               multiples of 4, else row by row by TMA gather4.
//   warp 1      TMEM allocator and the single MMA-issuing thread.
//   warps 2-5   softmax of query tile 0, warps 6-9 of query tile 1: each
//               thread owns one query row (TMEM lane 32*(warp mod 4) + lane).
//               In window calls the warpgroups shift by two warps (4-7, 8-11)
//               so that setmaxnreg can move registers from warpgroup 0 to them.
// TMEM (512 columns): S0 | S1 | O0 | O1, 128 fp32 columns each.  P (bf16)
// overwrites the first 64 columns of its S tile and feeds the PV MMA straight
// from TMEM.  P is handed over in two parts of 64 keys, each with its own
// barrier, so the PV product of the first part runs while the softmax
// computes the second.  Online softmax rescales O in TMEM only when some row of a warp
// sees its running maximum grow by more than 2^8 (the final normalisation uses
// the same stale maximum in numerator and denominator, so the result is exact).
// Window outputs are merged without atomics: the units of one parity class
// of windows never overlap, and the classes add into the fp32 accumulator
// rows of overlapped tokens one after another (see the epilogue).
// Every branch around a .sync.aligned tcgen05 instruction is warp-uniform.
// Every mbarrier wait is bounded (2 s of %globaltimer); on expiry the kernel
// records an error code, stops issuing work and still releases its TMEM.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "area_internal.cuh"

namespace area {

__device__ int g_tc_error = 0;   // set on a bounded-wait expiry; read by tests

namespace {

// Dense calls: 320 threads (producer, MMA issuer, 8 softmax warps), every
// thread at the block's register cap.  Window calls: 384 threads, warpgroup 0
// (producer, MMA issuer, two idle warps) drops to kRegsLow registers and the
// two softmax warpgroups rise to kRegsHigh; the split uses exactly the
// allocation of a 168-register launch (launch_tc checks it before launching).
__host__ __device__ constexpr int tc_threads(bool window) { return window ? 384 : 320; }
__host__ __device__ constexpr int tc_soft_warp0(bool window) { return window ? 4 : 2; }   // first softmax warp
constexpr int kRegsLow = 136, kRegsHigh = 184;
static_assert(128 * kRegsLow + 256 * kRegsHigh == 384 * 168, "register split");
constexpr int kStages = 4;               // K/V ring stages (32 KB each at head_dim 128)
constexpr int kQSlots = 1;               // query buffers (a second one would cost a K/V stage)
constexpr int kHalfBytes = 128 * 128;   // 128 rows x 64 bf16: one 128B-swizzled half tile
constexpr uint64_t kWaitNs = 2000000000ull;
constexpr float kRescaleThreshold = 8.0f;   // log2 units
constexpr int kMaxChains = 8;                // independent partial maxima of a score row
constexpr int kPParts = 2;                   // P handed to the PV product in this many parts
// Window keys and queries: patches and cells of the token grid (kPW x kPH,
// kCW x kCH; rect_tiling and window_query_token in area_internal.cuh).  A
// cell of one 64-column half takes kCellBytes of shared memory.
constexpr int kCellBytes = kCellKeys * 128;
static_assert(kCells <= 32 && kCellBytes % 1024 == 0, "cells: one lane each, whole swizzle atoms");
constexpr int kRecSlots = 3;                 // unit records in flight (shared-memory ring)

// Tile geometry for head_dim D (64 or 128): a tile is 128 rows of D bf16,
// stored as D / 64 halves of 64 columns, each the canonical K-major SW128
// layout of UMMA.  Shared-memory plan (offsets from a 1024-aligned base): the
// two Q tiles, the K/V ring, then the barriers.
template <int D>
struct Geo {
  static_assert(D == 64 || D == 128, "head_dim");
  static constexpr int kHalves = D / 64;
  static constexpr int kTileBytes = kHalves * kHalfBytes;
  static constexpr int kSmemQ = 0;                            // kQSlots x 2 query tiles
  static constexpr int kSmemKV = kQSlots * 2 * kTileBytes;
  static constexpr int kSmemBar = kSmemKV + kStages * kTileBytes;
  static constexpr int kSmemBytes = kSmemBar + 256 + 1024;   // barriers + alignment slack
  static_assert(kSmemBytes + 1024 <= 227 * 1024, "shared memory of one CTA");
};

// barrier indices
enum {
  BAR_Q_FULL = 0,                    // kQSlots of them
  BAR_Q_EMPTY = BAR_Q_FULL + kQSlots,
  BAR_S_FULL0 = BAR_Q_EMPTY + kQSlots, BAR_S_FULL1,
  BAR_P_FULL0, BAR_P_FULL1,
  BAR_O_FULL0, BAR_O_FULL1,
  BAR_P_PART0,                       // kPParts - 1 per query tile: leading parts of P stored
  BAR_P_PART1 = BAR_P_PART0 + kPParts - 1,
  BAR_KV_FULL = BAR_P_PART1 + kPParts - 1,  // kStages of them
  BAR_KV_EMPTY = BAR_KV_FULL + kStages,
  BAR_REC_FULL = BAR_KV_EMPTY + kStages,     // kRecSlots unit-record slots
  BAR_REC_EMPTY = BAR_REC_FULL + kRecSlots,
  BAR_DRAIN = BAR_REC_EMPTY + kRecSlots,     // MMA completion before TMEM release
  BAR_COUNT
};
static_assert(BAR_COUNT * 8 <= 256, "barrier area");

// ---------------------------------------------------------------------------
// PTX wrappers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
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

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Bounded wait for the phase of the given parity.  Returns false on expiry.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, int* abort_flag) {
  if (mbar_try(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  uint32_t it = 0;
  while (!mbar_try(bar, parity)) {
    if ((++it & 255u) == 0) {
      if (*(volatile int*)abort_flag) return false;
      if (global_ns() - t0 > kWaitNs) {
        *(volatile int*)abort_flag = 1;
        atomicExch(&g_tc_error, 1);
        return false;
      }
    }
  }
  return true;
}

// Lane 0 waits; the outcome is broadcast so the warp stays converged.
__device__ __forceinline__ bool warp_wait0(uint32_t bar, uint32_t parity, int* abort_flag) {
  int ok = 1;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, abort_flag) ? 1 : 0;
  return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

// Every lane waits (each acquires the barrier); the warp proceeds only if all
// lanes saw the phase complete, so `.sync.aligned` TMEM accesses stay converged.
__device__ __forceinline__ bool warp_wait_all(uint32_t bar, uint32_t parity, int* abort_flag) {
  const bool ok = mbar_wait(bar, parity, abort_flag);
  return __all_sync(0xffffffffu, ok) != 0;
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1)
      : "memory");
}

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

// Four rows (of a 2-D map) gathered into consecutive rows of shared memory.
__device__ __forceinline__ void tma_gather4(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int c0, int r0, int r1, int r2, int r3) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6, %7}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(r0), "r"(r1), "r"(r2),
      "r"(r3)
      : "memory");
}

// 16 bytes global -> shared, asynchronous (L2 only), and the arrive-on of an
// mbarrier when all of the thread's earlier cp.async copies have landed (the
// barrier's pending count is raised by one at once, so the phase cannot
// complete before the copies).
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
// 32-byte global accesses (sm_100): a thread moves one whole L2 sector per
// instruction.  The addresses must be 32-byte aligned.
__device__ __forceinline__ void st_global_v8(void* p, const uint32_t (&w)[8]) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(w[0]),
               "r"(w[1]), "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7])
               : "memory");
}
__device__ __forceinline__ void st_global_v8f(float* p, const float* f) {
  asm volatile("st.global.v8.f32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "f"(f[0]),
               "f"(f[1]), "f"(f[2]), "f"(f[3]), "f"(f[4]), "f"(f[5]), "f"(f[6]), "f"(f[7])
               : "memory");
}
__device__ __forceinline__ void ld_global_v8f(const float* p, float* f) {
  asm volatile("ld.global.v8.f32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=f"(f[0]), "=f"(f[1]), "=f"(f[2]), "=f"(f[3]), "=f"(f[4]), "=f"(f[5]),
                 "=f"(f[6]), "=f"(f[7])
               : "l"(p)
               : "memory");
}
__device__ __forceinline__ void cp_async_arrive(uint32_t bar) {
  asm volatile("cp.async.mbarrier.arrive.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}
// Shared-memory writes of the generic proxy (cp.async) made visible to the
// async proxy (tcgen05.mma operands).
__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// UMMA shared-memory descriptor, 128-byte swizzle, sm_100 version field.
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

// Instruction descriptors: fp32 accumulate, bf16 A and B, M = 128.  QK^T has
// N = 128 keys; PV has N = D with B (V) MN-major.
__host__ __device__ constexpr uint32_t idesc(uint32_t n, bool b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (b_mn_major ? (1u << 16) : 0u) | ((n >> 3) << 17) |
         ((128u >> 4) << 24);
}
constexpr uint32_t kIdescQK = idesc(128, false);

__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                       uint32_t accum) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(accum)
      : "memory");
}

__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b,
                                       uint32_t idesc, uint32_t accum) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b), "r"(idesc), "r"(accum)
      : "memory");
}

__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
      : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

#define AREA_R32(a) "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3]), "=r"(a[4]), "=r"(a[5]), \
  "=r"(a[6]), "=r"(a[7]), "=r"(a[8]), "=r"(a[9]), "=r"(a[10]), "=r"(a[11]), "=r"(a[12]),   \
  "=r"(a[13]), "=r"(a[14]), "=r"(a[15]), "=r"(a[16]), "=r"(a[17]), "=r"(a[18]),            \
  "=r"(a[19]), "=r"(a[20]), "=r"(a[21]), "=r"(a[22]), "=r"(a[23]), "=r"(a[24]),            \
  "=r"(a[25]), "=r"(a[26]), "=r"(a[27]), "=r"(a[28]), "=r"(a[29]), "=r"(a[30]), "=r"(a[31])
#define AREA_W32(a) "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(a[4]), "r"(a[5]),       \
  "r"(a[6]), "r"(a[7]), "r"(a[8]), "r"(a[9]), "r"(a[10]), "r"(a[11]), "r"(a[12]),          \
  "r"(a[13]), "r"(a[14]), "r"(a[15]), "r"(a[16]), "r"(a[17]), "r"(a[18]), "r"(a[19]),      \
  "r"(a[20]), "r"(a[21]), "r"(a[22]), "r"(a[23]), "r"(a[24]), "r"(a[25]), "r"(a[26]),      \
  "r"(a[27]), "r"(a[28]), "r"(a[29]), "r"(a[30]), "r"(a[31])

// 32 consecutive TMEM columns of this thread's lane.  The wait sits in the
// same asm statement, so no use of the registers can be scheduled before it.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
      "%28, %29, %30, %31}, [%32];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : AREA_R32(r)
      : "r"(taddr)
      : "memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, "
      "%10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, "
      "%27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      AREA_W32(r)
      : "memory");
}

// 128 consecutive TMEM columns of this thread's lane, loaded and waited for
// in one statement (one round trip per S or O tile).
__device__ __forceinline__ void tmem_ld128(uint32_t taddr, uint32_t (&r)[128]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x128.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, %48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63, %64, %65, %66, %67, %68, %69, %70, %71, %72, %73, %74, %75, %76, %77, %78, %79, %80, %81, %82, %83, %84, %85, %86, %87, %88, %89, %90, %91, %92, %93, %94, %95, %96, %97, %98, %99, %100, %101, %102, %103, %104, %105, %106, %107, %108, %109, %110, %111, %112, %113, %114, %115, %116, %117, %118, %119, %120, %121, %122, %123, %124, %125, %126, %127}, [%128];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]), "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]), "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63]), "=r"(r[64]), "=r"(r[65]), "=r"(r[66]), "=r"(r[67]), "=r"(r[68]), "=r"(r[69]), "=r"(r[70]), "=r"(r[71]), "=r"(r[72]), "=r"(r[73]), "=r"(r[74]), "=r"(r[75]), "=r"(r[76]), "=r"(r[77]), "=r"(r[78]), "=r"(r[79]), "=r"(r[80]), "=r"(r[81]), "=r"(r[82]), "=r"(r[83]), "=r"(r[84]), "=r"(r[85]), "=r"(r[86]), "=r"(r[87]), "=r"(r[88]), "=r"(r[89]), "=r"(r[90]), "=r"(r[91]), "=r"(r[92]), "=r"(r[93]), "=r"(r[94]), "=r"(r[95]), "=r"(r[96]), "=r"(r[97]), "=r"(r[98]), "=r"(r[99]), "=r"(r[100]), "=r"(r[101]), "=r"(r[102]), "=r"(r[103]), "=r"(r[104]), "=r"(r[105]), "=r"(r[106]), "=r"(r[107]), "=r"(r[108]), "=r"(r[109]), "=r"(r[110]), "=r"(r[111]), "=r"(r[112]), "=r"(r[113]), "=r"(r[114]), "=r"(r[115]), "=r"(r[116]), "=r"(r[117]), "=r"(r[118]), "=r"(r[119]), "=r"(r[120]), "=r"(r[121]), "=r"(r[122]), "=r"(r[123]), "=r"(r[124]), "=r"(r[125]), "=r"(r[126]), "=r"(r[127])
      : "r"(taddr)
      : "memory");
}

__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Packed fp32 pair arithmetic of sm_100 (one instruction for two lanes of work).
__device__ __forceinline__ void fma2(float& y0, float& y1, float a0, float a1, float b, float c) {
  asm("{\n\t.reg .b64 pa, pb, pc, pd;\n\t"
      "mov.b64 pa, {%2, %3};\n\tmov.b64 pb, {%4, %4};\n\tmov.b64 pc, {%5, %5};\n\t"
      "fma.rn.f32x2 pd, pa, pb, pc;\n\tmov.b64 {%0, %1}, pd;\n\t}"
      : "=f"(y0), "=f"(y1) : "f"(a0), "f"(a1), "f"(b), "f"(c));
}
__device__ __forceinline__ void add2(float& s0, float& s1, float a0, float a1) {
  asm("{\n\t.reg .b64 pa, ps;\n\t"
      "mov.b64 pa, {%2, %3};\n\tmov.b64 ps, {%0, %1};\n\t"
      "add.rn.f32x2 ps, ps, pa;\n\tmov.b64 {%0, %1}, ps;\n\t}"
      : "+f"(s0), "+f"(s1) : "f"(a0), "f"(a1));
}
__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
// ---------------------------------------------------------------------------
// Work units.  The producer warp turns each unit into a record in a
// kRecSlots-slot shared-memory ring (FULL: the producer wrote it; EMPTY: the
// MMA thread and the eight softmax warps are done with it).  Nobody else
// decodes the plan, so no role waits on a chain of dependent global loads at
// a unit boundary.
// ---------------------------------------------------------------------------
struct DenseArgs {
  int B, H, N, Nk;
  int units_per_head;   // ceil(N / 256)
};

struct UnitRec {
  int4 win, ext;      // window: the window and its Halo rectangle (y0, x0, hy, wx)
  int4 my, mx;        // window: merge geometry of the base window per axis (axis_merge)
  long long glist;    // window: element offset of the global list in the plan or cand
  int valid;          // 0: no more work for this CTA
  int bh, b;
  int q0;             // first query position of tile 0 (tile 1 = q0 + 128)
  int nq;             // valid query positions (dense: N; window: its area)
  int nkv;            // keys of the leading list tiles (dense keys, or global-KV count)
  int ngt;            // leading list tiles (dense key tiles, or global-KV tiles)
  int ntr;            // window: Halo-rectangle tiles, after the list tiles
  int qcx;            // window: cells per row of the window when its queries come
                      // in cells (sides multiples of kCH, kCW), else 0
  int nt;             // all key tiles of the unit, text tiles included
  int cls;            // window: parity class of the base window
  int one;            // 1: at most 128 valid queries, only query tile 0 runs
};
static_assert(sizeof(UnitRec) <= 128, "unit record");

// Tensor maps of one launch (bf16, 128B swizzle, boxes of 64 head dims).
struct TcMaps {
  CUtensorMap q;        // queries [rows, D]: 128-row box (dense), 1-row box (window gather4)
  CUtensorMap qc;       // window queries [B*H*Hg, Wg, D]: one cell
  CUtensorMap k, v;     // dense keys and values [rows, D]: 128-row box
  CUtensorMap kp, vp;   // window keys and values [B*H*Hg, Wg, D]: one patch
  CUtensorMap kc, vc;   // window keys and values [B*H*Hg, Wg, D]: one cell
  CUtensorMap kt, vt;   // text keys and values [B*H*T, D]: 128-row box
  CUtensorMap ks, vs;   // staged global-KV rows [B*H*nw*G, D]: 128-row box
};

struct TcParams {
  float scale_log2;
  int H;
  int T;              // text keys per (b, h), appended after the image keys
  const int* cand;    // bridge mode: per-head candidate tokens [B*H][R] (else null)
  int R;
  int num_units;      // dense: all units; window: capacity (the plan holds the count)
  DenseArgs da;
  PlanView P;
  __nv_bfloat16* o;   // output
  const __nv_bfloat16 *k, *v;       // window: keys and values, for rows copied with cp.async
  unsigned* counters; // window: workspace header (unit counter, per-class completions)
  float* acc;         // window: fp32 accumulator rows [B*H][n_ov][128]
  int nx2;            // window: columns covered by two base windows
  long long n_ov;     // window: overlapped tokens per element
  int staged;         // window: whole global-KV tiles come from the staging area
};


// One 128-row tile of D bf16 copied row by row with cp.async by the 32 lanes
// of a warp into the 128B-swizzled K-major layout that TMA's 128-byte swizzle
// produces (and UMMA reads): in each 64-column half, row R at R * 128 bytes,
// its 16-byte chunk c at ((c ^ (R mod 8)) * 16).  Lane l holds the source
// rows of tile rows 4l .. 4l + 3 in r[0..3] (row indices of `base`).  Each
// warp instruction copies whole rows (256 or 128 contiguous bytes per row).
// Gathered global-KV rows go this way rather than through tile::gather4,
// whose issue rate (about 7 bytes per clock per SM, measured) made them the
// window kernel's largest fixed cost.  Used for rows that are mostly in L2
// (the global-KV lists); for rows read from DRAM a warp's cp.async stream
// keeps too few reads in flight, and TMA gather4 does better.
template <int D>
__device__ __forceinline__ void cp_async_rows(uint32_t dst, const __nv_bfloat16* base,
                                              const int (&r)[4], int lane) {
  constexpr int kChunks = D / 8;              // 16-byte chunks per row: 16 or 8
  constexpr int kRowsPerIt = 32 / kChunks;    // rows per warp instruction: 2 or 4
  const int q = lane % kChunks, sub = lane / kChunks;
  const uint32_t half = (uint32_t)((q >> 3) * kHalfBytes);
  const int c = q & 7;
#pragma unroll 4
  for (int o = 0; o < 32; ++o) {              // the four rows held by lane o
    const int t0 = __shfl_sync(0xffffffffu, r[0], o), t1 = __shfl_sync(0xffffffffu, r[1], o);
    const int t2 = __shfl_sync(0xffffffffu, r[2], o), t3 = __shfl_sync(0xffffffffu, r[3], o);
#pragma unroll
    for (int k = 0; k < 4 / kRowsPerIt; ++k) {
      const int e = k * kRowsPerIt + sub;     // which of the four
      const int tok = e == 0 ? t0 : e == 1 ? t1 : e == 2 ? t2 : t3;
      const int R = o * 4 + e;
      cp_async16(dst + half + (uint32_t)(R * 128 + ((c ^ (R & 7)) << 4)),
                 base + (int64_t)tok * D + q * 8);
    }
  }
}

// The record of work item idx of batch element b for head h.
__device__ void fill_window_unit(int b, int h, int idx, const TcParams& prm, UnitRec& r) {
  const PlanView& P = prm.P;
  const int2 it = P.items[(int64_t)b * P.nitem_max + idx];
  const int64_t wo = (int64_t)b * P.nw + it.x;
  r.b = b;
  r.bh = b * prm.H + h;
  r.win = P.win[wo];
  r.ext = P.ext[wo];
  const int parent = P.parent[wo];
  r.cls = window_class(parent, P.nbx);
  r.my = axis_merge(parent / P.nbx, P.nby, P.Hg, P.hy, P.sy);
  r.mx = axis_merge(parent % P.nbx, P.nbx, P.Wg, P.wx, P.sx);
  r.q0 = it.y * 256;
  r.nq = r.win.z * r.win.w;
  r.one = r.nq - r.q0 <= 128;
  r.nkv = prm.cand ? prm.R : P.gcount[wo];
  r.ngt = (r.nkv + 127) / 128;
  r.ntr = rect_tiles(rect_tiling(r.ext.z, r.ext.w));
  r.qcx = query_cells_per_row(r.win);
  r.nt = r.ngt + r.ntr + (prm.T + 127) / 128;
  r.glist = prm.cand ? (long long)r.bh * prm.R : (long long)wo * P.G;
}

// Decode unit u into a record (producer lane 0).  Dense: (b*H + h, 256-query
// block), head-major.  Window: by parity class, then batch element, then
// head, then the class's work items in plan order (unsplit windows first,
// costliest first).  A class's units all come before the next class's, so a
// unit merging into an overlapped token rarely waits for the earlier class;
// with few units per head a head-by-head order made the classes wait on each
// other (measured), so the order is class-major over all heads.
template <bool WINDOW>
__device__ bool decode_unit(int u, const TcParams& prm, UnitRec& r) {
  r.valid = 1;
  r.one = 0;
  r.cls = 0;
  r.glist = 0;
  r.ntr = r.qcx = 0;
  r.win = r.ext = r.my = r.mx = make_int4(0, 0, 0, 0);
  if (!WINDOW) {
    if (u >= prm.num_units) return false;
    r.bh = u / prm.da.units_per_head;
    r.b = r.bh / prm.da.H;
    r.q0 = (u % prm.da.units_per_head) * 256;
    r.nq = prm.da.N;
    r.one = r.nq - r.q0 <= 128;
    r.nkv = prm.da.Nk;
    r.ngt = (prm.da.Nk + 127) / 128;
    r.nt = r.ngt + (prm.T + 127) / 128;
    return true;
  }
  const PlanView& P = prm.P;
  int rem = u;
  for (int c = 0; c < 4; ++c)
    for (int b = 0; b < P.B; ++b) {
      const int n = P.nclass[b * 4 + c];
      if (rem >= n * prm.H) {
        rem -= n * prm.H;
        continue;
      }
      int coff = 0;                          // the class's first item (items are class by class)
      for (int c2 = 0; c2 < c; ++c2) coff += P.nclass[b * 4 + c2];
      fill_window_unit(b, rem / n, coff + rem % n, prm, r);
      return true;
    }
  return false;
}

template <bool WINDOW, bool BRIDGE, int D>
__global__ void __launch_bounds__(tc_threads(WINDOW), 1)
attn_tc_kernel(const __grid_constant__ TcMaps tm, const TcParams prm) {
  using G = Geo<D>;
  constexpr int kSoftWarp0 = tc_soft_warp0(WINDOW);
  constexpr uint32_t kIdescPV = idesc(D, true);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + G::kSmemBar;
  __shared__ uint32_t s_tmem_base;
  __shared__ int s_abort;
  __shared__ __align__(16) UnitRec s_rec[kRecSlots];
  auto bar = [&](int i) { return bar0 + 8u * (uint32_t)i; };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    s_abort = 0;
    for (int q = 0; q < kQSlots; ++q) {
      mbar_init(bar(BAR_Q_FULL + q), 1);
      mbar_init(bar(BAR_Q_EMPTY + q), 1);
    }
    mbar_init(bar(BAR_S_FULL0), 1);
    mbar_init(bar(BAR_S_FULL1), 1);
    mbar_init(bar(BAR_P_FULL0), 128);
    mbar_init(bar(BAR_P_FULL1), 128);
    for (int h = 0; h < kPParts - 1; ++h) {
      mbar_init(bar(BAR_P_PART0 + h), 128);
      mbar_init(bar(BAR_P_PART1 + h), 128);
    }
    mbar_init(bar(BAR_O_FULL0), 1);
    mbar_init(bar(BAR_O_FULL1), 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar(BAR_KV_FULL + s), 1);
      mbar_init(bar(BAR_KV_EMPTY + s), 1);
    }
    for (int s = 0; s < kRecSlots; ++s) {
      mbar_init(bar(BAR_REC_FULL + s), 1);
      mbar_init(bar(BAR_REC_EMPTY + s), 9);   // the MMA thread and the 8 softmax warps
    }
    mbar_init(bar(BAR_DRAIN), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(
                     smem_u32(&s_tmem_base))
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem_base;
  int* abort_flag = &s_abort;
  const int Wg = WINDOW ? prm.P.Wg : 0;
  const int Ntok = WINDOW ? prm.P.N : prm.da.N;     // rows per (b, h) of Q
  const int Nkrows = WINDOW ? prm.P.N : prm.da.Nk;  // rows per (b, h) of K and V

  if (warp < kSoftWarp0) {
    // warpgroup 0 (window calls: producer, MMA issuer, two idle warps)
    if constexpr (WINDOW) asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsLow) : "memory");
    if (warp == 0) {
      // ------------------------------------------------------------ producer
      // Units are claimed from a counter in the workspace (window mode) or
      // statically (dense mode).  The record of the next unit is written while
      // the current unit's first key tiles are in flight.
      uint32_t kv_it = 0, unit_count = 0, claims = 0;
      bool ok = true;
      auto claim = [&]() -> int {
        int u = 0;
        if (lane == 0) {
          if (WINDOW) u = (int)atomicAdd(prm.counters + kWsUnitCounter, 1u);
          else u = blockIdx.x + (int)claims * gridDim.x;
        }
        ++claims;
        return __shfl_sync(0xffffffffu, u, 0);
      };
      // Claim, decode and publish the record of this CTA's k-th unit.
      auto publish = [&](uint32_t k) -> bool {
        const int u = claim();
        const uint32_t slot = k % kRecSlots;
        if (!warp_wait0(bar(BAR_REC_EMPTY + slot), ((k / kRecSlots) & 1u) ^ 1u, abort_flag))
          return false;
        if (lane == 0) {
          UnitRec r;
          if (!decode_unit<WINDOW>(u, prm, r)) r.valid = 0;
          s_rec[slot] = r;
          mbar_arrive(bar(BAR_REC_FULL + slot));
        }
        __syncwarp();
        return true;
      };
      // Queries of this CTA's k-th unit, once the previous unit's last QK has
      // read the buffer.  Window queries are read from DRAM once per unit: in
      // cells of kCW x kCH tokens (one tiled box per lane) when the window's
      // sides allow, else row by row with TMA gather4, 4 rows per lane (a warp's
      // cp.async stream issued those about 7x slower, measured; gather4 itself
      // moves about 7 bytes per clock per SM against about 37 for tiled boxes).
      auto load_q = [&](uint32_t k) -> bool {
        const UnitRec& Rq = s_rec[k % kRecSlots];
        if (!Rq.valid) return true;
        const uint32_t qs = k % kQSlots;
        if (!warp_wait0(bar(BAR_Q_EMPTY + qs), ((k / kQSlots) & 1u) ^ 1u, abort_flag)) return false;
        const uint32_t qbase = sbase + G::kSmemQ + qs * 2 * G::kTileBytes;
        const int nqt = Rq.one ? 1 : 2;
        if constexpr (!WINDOW) {
          if (lane == 0) {
            mbar_arrive_tx(bar(BAR_Q_FULL + qs), nqt * G::kTileBytes);
            for (int t = 0; t < nqt; ++t)
              for (int hf = 0; hf < G::kHalves; ++hf)
                tma_load_2d(qbase + t * G::kTileBytes + hf * kHalfBytes, &tm.q, bar(BAR_Q_FULL + qs),
                            hf * 64, Rq.bh * Ntok + Rq.q0 + t * 128);
          }
          __syncwarp();
        } else if (Rq.qcx > 0) {
          if (lane == 0) mbar_arrive_tx(bar(BAR_Q_FULL + qs), nqt * G::kTileBytes);
          __syncwarp();
          if (lane < kCells) {
            // cell q0 / kCellKeys + t * kCells + lane (clamped to the last one;
            // the rows past nq are computed and not stored)
            const int ncq = Rq.nq / kCellKeys;
            for (int t = 0; t < nqt; ++t) {
              int c = Rq.q0 / kCellKeys + t * kCells + lane;
              if (c > ncq - 1) c = ncq - 1;
              const int cx = Rq.win.y + (c % Rq.qcx) * kCW;
              const int cy = Rq.bh * prm.P.Hg + Rq.win.x + (c / Rq.qcx) * kCH;
              for (int hf = 0; hf < G::kHalves; ++hf)
                tma_load_3d(qbase + t * G::kTileBytes + hf * kHalfBytes + lane * kCellBytes, &tm.qc,
                            bar(BAR_Q_FULL + qs), hf * 64, cx, cy);
            }
          }
          __syncwarp();
        } else {
          if (lane == 0) mbar_arrive_tx(bar(BAR_Q_FULL + qs), nqt * G::kTileBytes);
          __syncwarp();
          for (int t = 0; t < nqt; ++t) {
            int r[4];
  #pragma unroll
            for (int i = 0; i < 4; ++i)
              r[i] = Rq.bh * Ntok +
                     window_query_token(Rq.win, 0, Rq.nq, Rq.q0 + t * 128 + lane * 4 + i, Wg);
            for (int hf = 0; hf < G::kHalves; ++hf)
              tma_gather4(qbase + t * G::kTileBytes + hf * kHalfBytes + lane * 512, &tm.q,
                          bar(BAR_Q_FULL + qs), hf * 64, r[0], r[1], r[2], r[3]);
          }
        }
        return true;
      };
      ok = publish(0);
      while (ok) {
        const UnitRec& R = s_rec[unit_count % kRecSlots];
        if (!R.valid) break;
        if (!(ok = load_q(unit_count))) break;
        const int nt = R.nt, ngt = R.ngt, ntr = R.ntr, nkv = R.nkv;
        const int nti = ngt + ntr;
        const int bh = R.bh;
        const int4 ext = R.ext;
        const RectTiling rt = rect_tiling(ext.z, ext.w);
        const int* glist = (BRIDGE ? prm.cand : prm.P.gidx) + R.glist;
        const int jn = nt < 2 ? nt : 2;         // the next record is published before tile jn
        bool published = false;
        for (int j = 0; j < nt && ok; ++j) {
          if (j == jn) {
            published = true;
            if (!(ok = publish(unit_count + 1))) break;
          }
          for (int kv = 0; kv < 2; ++kv) {       // K then V
            const int s = (int)(kv_it % kStages);
            if (!warp_wait0(bar(BAR_KV_EMPTY + s), ((kv_it / kStages) & 1u) ^ 1u, abort_flag)) {
              ok = false;
              break;
            }
            const CUtensorMap* tmd = kv ? &tm.v : &tm.k;
            const uint32_t dst = sbase + G::kSmemKV + s * G::kTileBytes;
            if (WINDOW && j < ngt && prm.staged && (j + 1) * 128 <= nkv) {
              // a whole tile of the window's global-KV rows (or of the head's
              // bridge candidates), staged in the workspace by this call's copy
              // launch: one tiled load
              if (lane == 0) {
                mbar_arrive_tx(bar(BAR_KV_FULL + s), G::kTileBytes);
                // staging row: plan lists ((b * H + h) * nw + w) * G with
                // R.glist = (b * nw + w) * G; candidates (b * H + h) * R = R.glist
                const long long srow =
                    BRIDGE ? R.glist : R.glist + (long long)(bh - R.b) * prm.P.nw * prm.P.G;
                for (int hf = 0; hf < G::kHalves; ++hf)
                  tma_load_2d(dst + hf * kHalfBytes, kv ? &tm.vs : &tm.ks, bar(BAR_KV_FULL + s),
                              hf * 64, (int)(srow + j * 128));
              }
              __syncwarp();
              ++kv_it;
              continue;
            }
            if (WINDOW && j < ngt) {
              // global-KV list (or bridge candidates), copied row by row: the
              // rows of a head's list serve all its windows and sit in L2, and
              // from L2 cp.async beats TMA gather4 by about 4x (measured)
              const int g0 = j * 128 + lane * 4;
              int r[4];
  #pragma unroll
              for (int i = 0; i < 4; ++i) {
                const int p = g0 + i < nkv ? g0 + i : nkv - 1;
                r[i] = bh * Nkrows + glist[p];
              }
              cp_async_rows<D>(dst, kv ? prm.v : prm.k, r, lane);
              cp_async_arrive(bar(BAR_KV_FULL + s));
              __syncwarp();
              if (lane == 0) mbar_arrive(bar(BAR_KV_FULL + s));
              ++kv_it;
              continue;
            }
            if (lane == 0) mbar_arrive_tx(bar(BAR_KV_FULL + s), G::kTileBytes);
            __syncwarp();
            if (j >= nti) {
              // text keys: rows of the [B*H*T, 128] text tensors
              if (lane == 0) {
                const CUtensorMap* tt = kv ? &tm.vt : &tm.kt;
                for (int hf = 0; hf < G::kHalves; ++hf)
                  tma_load_2d(dst + hf * kHalfBytes, tt, bar(BAR_KV_FULL + s), hf * 64,
                              bh * prm.T + (j - nti) * 128);
              }
            } else if (!WINDOW) {
              if (lane == 0)
                for (int hf = 0; hf < G::kHalves; ++hf)
                  tma_load_2d(dst + hf * kHalfBytes, tmd, bar(BAR_KV_FULL + s), hf * 64,
                              bh * Nkrows + j * 128);
            } else {
              // Halo rectangle: patch j - ngt, or kCells strip cells, one per
              // lane (past the last cell the last one is loaded again: finite
              // values under masked keys)
              const int jj = j - ngt;
              if (jj < rt.npatch) {
                if (lane == 0) {
                  const CUtensorMap* tp = kv ? &tm.vp : &tm.kp;
                  const int cx = ext.y + (jj % rt.npx) * kPW;
                  const int cy = bh * prm.P.Hg + ext.x + (jj / rt.npx) * kPH;
                  for (int hf = 0; hf < G::kHalves; ++hf)
                    tma_load_3d(dst + hf * kHalfBytes, tp, bar(BAR_KV_FULL + s), hf * 64, cx, cy);
                }
              } else if (lane < kCells) {
                const CUtensorMap* tc = kv ? &tm.vc : &tm.kc;
                int c = (jj - rt.npatch) * kCells + lane;
                if (c > rt.ncell - 1) c = rt.ncell - 1;
                const int2 o = strip_cell(rt, c);
                const int cx = ext.y + o.y;
                const int cy = bh * prm.P.Hg + ext.x + o.x;
                for (int hf = 0; hf < G::kHalves; ++hf)
                  tma_load_3d(dst + hf * kHalfBytes + lane * kCellBytes, tc, bar(BAR_KV_FULL + s),
                              hf * 64, cx, cy);
              }
              __syncwarp();
            }
            ++kv_it;
          }
        }
        if (!ok) break;
        if (!published && !(ok = publish(unit_count + 1))) break;
        ++unit_count;
      }
      // Drain: the most recent load of every stage has landed (bounded wait),
      // and no cp.async copy of this warp is still in flight.
      int drain_abort = 0;
      for (uint32_t k = 0; k < kStages && k < kv_it; ++k) {
        const uint32_t it = kv_it - 1 - k;
        warp_wait0(bar(BAR_KV_FULL + it % kStages), (it / kStages) & 1u, &drain_abort);
      }
      asm volatile("cp.async.wait_all;" ::: "memory");
    } else if (warp == 1) {
      // ------------------------------------------------------------ MMA issuer
      if (lane == 0) {
        uint32_t kv_it = 0, unit_count = 0;
        uint32_t p_cnt0 = 0, p_cnt1 = 0;
        const uint32_t tS0 = tmem, tS1 = tmem + 128, tO0 = tmem + 256, tO1 = tmem + 384;

        bool ok = true;
        auto kv_addr = [&](uint32_t it) { return sbase + G::kSmemKV + (it % kStages) * G::kTileBytes; };
        auto qk = [&](uint32_t d, uint32_t qs, uint32_t ks) {
  #pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
            mma_ss(d, sdesc(qs + off, 16, 1024), sdesc(ks + off, 16, 1024), kIdescQK, kk > 0);
          }
        };
        // PV over part h of the tile's keys (128 / kPParts keys, 16 per instruction)
        auto pv_part = [&](uint32_t d, uint32_t p_tmem, uint32_t vs, bool first, int h) {
          constexpr int kPer = 8 / kPParts;
  #pragma unroll
          for (int kk = kPer * h; kk < kPer * h + kPer; ++kk)
            mma_ts(d, p_tmem + kk * 8, sdesc(vs + kk * 2048, kHalfBytes, 1024), kIdescPV,
                   (first && kk == 0) ? 0u : 1u);
        };
        // PV of one query tile, part by part as the softmax hands P over
        auto pv_parts = [&](uint32_t d, uint32_t p_tmem, uint32_t vs, bool first, int bpart,
                            int bfull, uint32_t cnt) {
  #pragma unroll
          for (int h = 0; h < kPParts; ++h) {
            const uint32_t b = h + 1 < kPParts ? bar(bpart + h) : bar(bfull);
            if (!mbar_wait(b, cnt & 1u, abort_flag)) return false;
            tc_fence_after();
            pv_part(d, p_tmem, vs, first, h);
          }
          return true;
        };
        while (ok) {
          const uint32_t slot = unit_count % kRecSlots;
          if (!(ok = mbar_wait(bar(BAR_REC_FULL + slot), (unit_count / kRecSlots) & 1u, abort_flag)))
            break;
          const int valid = s_rec[slot].valid, nt = s_rec[slot].nt;
          // leading list tiles copied by cp.async (not the staged whole ones)
          const int ngt = WINDOW ? s_rec[slot].ngt : 0;
          const int ncp = !WINDOW ? 0 : prm.staged ? ngt - s_rec[slot].nkv / 128 : ngt;
          auto copied = [&](int j) { return j < ngt && j >= ngt - ncp; };
          const bool two = s_rec[slot].one == 0;   // query tile 1 runs too
          mbar_arrive(bar(BAR_REC_EMPTY + slot));
          if (!valid) break;
          const uint32_t qs = unit_count % kQSlots;
          const uint32_t q0s = sbase + G::kSmemQ + qs * 2 * G::kTileBytes;
          const uint32_t q1s = q0s + G::kTileBytes;
          const uint32_t bQe = bar(BAR_Q_EMPTY + qs);
          if (!(ok = mbar_wait(bar(BAR_Q_FULL + qs), (unit_count / kQSlots) & 1u, abort_flag))) break;
          // prologue: S(0)
          const uint32_t k0 = kv_it;
          if (!(ok = mbar_wait(bar(BAR_KV_FULL + k0 % kStages), (k0 / kStages) & 1u, abort_flag)))
            break;
          if (copied(0)) fence_proxy_async();     // rows copied by cp.async
          tc_fence_after();
          qk(tS0, q0s, kv_addr(k0));
          mma_commit(bar(BAR_S_FULL0));
          if (two) {
            qk(tS1, q1s, kv_addr(k0));
            mma_commit(bar(BAR_S_FULL1));
          }
          mma_commit(bar(BAR_KV_EMPTY + k0 % kStages));
          if (nt == 1) mma_commit(bQe);
          for (int j = 0; j < nt && ok; ++j) {
            const uint32_t vi = kv_it + 2 * j + 1;
            const uint32_t kn = kv_it + 2 * j + 2;
            if (!(ok = mbar_wait(bar(BAR_KV_FULL + vi % kStages), (vi / kStages) & 1u, abort_flag)))
              break;
            if (copied(j)) fence_proxy_async();
            if (!(ok = pv_parts(tO0, tS0, kv_addr(vi), j == 0, BAR_P_PART0, BAR_P_FULL0, p_cnt0)))
              break;
            ++p_cnt0;
            if (j == nt - 1) mma_commit(bar(BAR_O_FULL0));
            if (j + 1 < nt) {
              if (!(ok = mbar_wait(bar(BAR_KV_FULL + kn % kStages), (kn / kStages) & 1u,
                                   abort_flag)))
                break;
              if (copied(j + 1)) fence_proxy_async();
              tc_fence_after();
              qk(tS0, q0s, kv_addr(kn));
              mma_commit(bar(BAR_S_FULL0));
              if (!two) {                          // K(j+1) is done with after QK0
                mma_commit(bar(BAR_KV_EMPTY + kn % kStages));
                if (j + 2 == nt) mma_commit(bQe);
              }
            }
            if (two) {
              if (!(ok = pv_parts(tO1, tS1, kv_addr(vi), j == 0, BAR_P_PART1, BAR_P_FULL1, p_cnt1)))
                break;
              ++p_cnt1;
              if (j == nt - 1) mma_commit(bar(BAR_O_FULL1));
            }
            mma_commit(bar(BAR_KV_EMPTY + vi % kStages));
            if (two && j + 1 < nt) {
              qk(tS1, q1s, kv_addr(kn));
              mma_commit(bar(BAR_S_FULL1));
              mma_commit(bar(BAR_KV_EMPTY + kn % kStages));
              if (j + 2 == nt) mma_commit(bQe);
            }
          }
          kv_it += 2 * nt;
          ++unit_count;
        }
        // Drain: every MMA issued by this thread has completed (bounded wait).
        int drain_abort = 0;
        mma_commit(bar(BAR_DRAIN));
        mbar_wait(bar(BAR_DRAIN), 0, &drain_abort);
      }
      __syncwarp();
    }
  } else {
    if constexpr (WINDOW) asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsHigh) : "memory");
    // ------------------------------------------------------------ softmax / epilogue
    // The first four softmax warps own query tile 0, the next four query
    // tile 1.  A warp may only touch the TMEM lane quarter (warp id mod 4),
    // and each group of four consecutive warps covers all four quarters.
    const int qt = (warp - kSoftWarp0) >> 2;         // query tile of this warpgroup
    const int row = ((warp & 3) << 5) + lane;        // TMEM lane = query row in the tile
    const uint32_t lane_off = (uint32_t)((warp & 3) << 5) << 16;
    const uint32_t tS = tmem + lane_off + (qt ? 128u : 0u);
    const uint32_t tO = tmem + lane_off + (qt ? 384u : 256u);
    const uint32_t bS = bar(qt ? BAR_S_FULL1 : BAR_S_FULL0);
    const uint32_t bP = bar(qt ? BAR_P_FULL1 : BAR_P_FULL0);
    const int bPpart = qt ? BAR_P_PART1 : BAR_P_PART0;
    const uint32_t bO = bar(qt ? BAR_O_FULL1 : BAR_O_FULL0);
    uint32_t s_cnt = 0, o_cnt = 0, unit_count = 0;
    const float sl2 = prm.scale_log2;
    bool ok = true;
    while (ok) {
      const uint32_t slot = unit_count % kRecSlots;
      if (!(ok = warp_wait_all(bar(BAR_REC_FULL + slot), (unit_count / kRecSlots) & 1u,
                               abort_flag)))
        break;
      const UnitRec& R = s_rec[slot];
      if (!R.valid) break;
      if (qt == 1 && R.one) {
        // at most 128 valid queries: query tile 1 does not run; its warps
        // only sign the unit off (completion count and record slot)
        if (WINDOW && lane == 0) atomicAdd(prm.counters + kWsClassDone + R.bh * 4 + R.cls, 1u);
        if (lane == 0) mbar_arrive(bar(BAR_REC_EMPTY + slot));
        ++unit_count;
        continue;
      }
      const int nkv = R.nkv, nt = R.nt, ngt = R.ngt, ntr = R.ntr;
      const int nti = ngt + ntr;
      const int ew = R.ext.w, eh = R.ext.z;
      int ncb, ncell;                                // first strip-cell tile, strip cells
      {
        const RectTiling rt = rect_tiling(eh, ew);
        ncb = ngt + rt.npatch;
        ncell = rt.ncell;
      }
      // a Halo rectangle whose sides are multiples of the cell's has full
      // cells only: its cell tiles hold a prefix of valid keys
      const bool ragged = WINDOW && (ew % kCW != 0 || eh % kCH != 0);
      float m = -INFINITY, l = 0.f;
      for (int j = 0; j < nt; ++j) {
        // Bridge candidates: drop those past the list or inside the Halo
        // rectangle; lane l tests keys 4l..4l+3 and ballots the result.  This
        // does not depend on S, so it is done before waiting for S (the loads
        // overlap the wait) and before S occupies 128 registers.  Keys of a
        // ragged rectangle's cells are tested the same way.
        const bool bridge_tile = BRIDGE && j < ngt;
        const bool ragged_tile = ragged && j >= ncb && j < nti;
        uint32_t keep[4] = {0xffffffffu, 0xffffffffu, 0xffffffffu, 0xffffffffu};
        if (bridge_tile || ragged_tile) {
          const int4 ex = R.ext;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int kk = lane * 4 + i;
            bool in;
            if (bridge_tile) {
              const int p = j * 128 + kk;
              in = p < nkv;
              if (in) {
                const int tok = prm.cand[R.glist + p];
                const int ty = tok / prm.P.Wg, tx = tok % prm.P.Wg;
                in = !(ty >= ex.x && ty < ex.x + ex.z && tx >= ex.y && tx < ex.y + ex.w);
              }
            } else {
              // the tiling is recomputed from the record here (a shared-memory
              // read the compiler cannot hoist past the loop's barrier waits)
              // rather than kept in registers through the whole tile loop
              const int c = (j - ncb) * kCells + kk / kCellKeys, e = kk % kCellKeys;
              in = c < ncell;
              if (in) {
                const int2 o = strip_cell(rect_tiling(ex.z, ex.w), c);
                in = o.y + e % kCW < ex.w && o.x + e / kCW < ex.z;
              }
            }
            keep[i] = __ballot_sync(0xffffffffu, in);
          }
        }
        if (!(ok = warp_wait_all(bS, s_cnt & 1u, abort_flag))) break;
        ++s_cnt;
        tc_fence_after();
        // Key validity (warp-uniform): bridge and ragged-rectangle tiles
        // follow their ballots (key k in bit k / 4 of keep[k % 4]), applied
        // to S in TMEM 32 columns at a time, so the ballots are not held
        // with the whole score row; list, text and rectangle tiles are a
        // prefix of `valid` keys.
        if (bridge_tile || ragged_tile) {
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            uint32_t t[32];
            tmem_ld32(tS + c * 32, t);
            const uint32_t k0 = keep[0], k1 = keep[1], k2 = keep[2], k3 = keep[3];
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const uint32_t kw = (i & 3) == 0 ? k0 : (i & 3) == 1 ? k1 : (i & 3) == 2 ? k2 : k3;
              if (!((kw >> (c * 8 + (i >> 2))) & 1u)) t[i] = 0xff800000u;
            }
            tmem_st32(tS + c * 32, t);
          }
          tmem_wait_st();
        }
        uint32_t sr[128];
        tmem_ld128(tS, sr);
        if (!(bridge_tile || ragged_tile)) {
          const int valid = j < ngt    ? min(128, nkv - j * 128)
                            : j < ncb  ? 128
                            : j < nti  ? min(128, (ncell - (j - ncb) * kCells) * kCellKeys)
                                       : min(128, prm.T - (j - nti) * 128);
          if (valid < 128) {
#pragma unroll
            for (int i = 0; i < 128; ++i)
              if (i >= valid) sr[i] = 0xff800000u;        // -inf: no weight
          }
        }
        // row maximum: kMaxChains independent partial maxima, then a tree
        float pm[kMaxChains];
#pragma unroll
        for (int t = 0; t < kMaxChains; ++t) pm[t] = __uint_as_float(sr[t]);
#pragma unroll
        for (int i = kMaxChains; i < 128; i += 2)
          pm[(i >> 1) % kMaxChains] = max3(pm[(i >> 1) % kMaxChains],
                                                __uint_as_float(sr[i]), __uint_as_float(sr[i + 1]));
#pragma unroll
        for (int t = kMaxChains / 2; t > 0; t >>= 1)
#pragma unroll
          for (int q = 0; q < t; ++q) pm[q] = fmaxf(pm[q], pm[q + t]);
        const float mx = pm[0];
        const float mnew = fmaxf(mx * sl2, m);
        // Rescale O only when some row of the warp gained more than 2^8; the
        // decision is warp-uniform because the TMEM accesses are .sync.aligned.
        // A row whose earlier keys were all masked has m = -inf (its l and O
        // are zero): it takes alpha = 0.
        const bool rescale = j > 0 && __any_sync(0xffffffffu, mnew > m + kRescaleThreshold);
        const float alpha = rescale ? (m == -INFINITY ? 0.f : fast_exp2(m - mnew)) : 1.f;
        if (j == 0 || rescale) m = mnew;
        l *= alpha;
        // P = exp2(S * scale * log2(e) - m) as bf16, two keys per TMEM column,
        // packed in place into sr[0..63] (slot i/2 was already read).  The
        // first 64 keys go out first, so the PV product can start on them
        // while the second 64 are computed; O is rescaled before that first
        // hand-over, so the PV products of this tile accumulate onto it.
        // While every key so far is masked (m = -inf) the reference is 0.
        float ls[4] = {0.f, 0.f, 0.f, 0.f};
        const float negm = m == -INFINITY ? 0.f : -m;
#pragma unroll
        for (int h = 0; h < kPParts; ++h) {
          constexpr int kKeys = 128 / kPParts;
#pragma unroll
          for (int i = kKeys * h; i < kKeys * h + kKeys; i += 2) {
            float x0, x1;
            fma2(x0, x1, __uint_as_float(sr[i]), __uint_as_float(sr[i + 1]), sl2, negm);
            const float p0 = fast_exp2(x0);
            const float p1 = fast_exp2(x1);
            if ((i >> 1) & 1) add2(ls[2], ls[3], p0, p1); else add2(ls[0], ls[1], p0, p1);
            sr[i >> 1] = pack_bf16(p0, p1);
          }
          if (h == 0 && rescale) {
#pragma unroll 1
            for (int c = 0; c < D / 32; ++c) {
              uint32_t orr[32];
              tmem_ld32(tO + c * 32, orr);
#pragma unroll
              for (int i = 0; i < 32; ++i)
                orr[i] = __float_as_uint(__uint_as_float(orr[i]) * alpha);
              tmem_st32(tO + c * 32, orr);
            }
          }
          tmem_st32(tS + 32 * h, *reinterpret_cast<const uint32_t(*)[32]>(&sr[32 * h]));
          tmem_wait_st();
          tc_fence_before();
          mbar_arrive(h + 1 < kPParts ? bar(bPpart + h) : bP);
        }
        l += (ls[0] + ls[1]) + (ls[2] + ls[3]);
      }
      if (!ok) break;
      // ---- epilogue
      const int qpos = R.q0 + qt * 128 + row;
      const bool qvalid = qpos < R.nq;
      const int bh = R.bh;
      if constexpr (!WINDOW) {
        if (!(ok = warp_wait_all(bO, o_cnt & 1u, abort_flag))) break;
        ++o_cnt;
        tc_fence_after();
        const float inv = 1.f / l;
        __nv_bfloat16* dst = prm.o + ((int64_t)bh * Ntok + qpos) * D;
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t orr[32];
          tmem_ld32(tO + c * 32, orr);
          if (qvalid) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              uint32_t w[8];
#pragma unroll
              for (int i = 0; i < 8; ++i)
                w[i] = pack_bf16(__uint_as_float(orr[16 * h + 2 * i]) * inv,
                                 __uint_as_float(orr[16 * h + 2 * i + 1]) * inv);
              st_global_v8(dst + c * 32 + h * 16, w);
            }
          }
        }
      } else {
        // Centre-weighted merge.  A token inside one window stores its output
        // directly.  A token in an overlap has one fp32 accumulator row: the
        // window of its lowest parity class stores t * O, the middle classes
        // add, the highest class adds and divides by the weight sum.  Windows
        // of one class never overlap, and a class adds only after every unit
        // of the lower classes has completed (a bounded wait on their
        // completion counters), so the sum runs in a fixed order.
        const int tok = window_query_token(R.win, R.qcx, R.nq, qpos, Wg);
        const int y = tok / Wg, x = tok % Wg;
        const MergeRole mr = merge_role(y, x, R.cls, R.my, R.mx, Wg, prm.nx2);
        const bool rmw = qvalid && mr.ov;
        // read before the O wait, so its latency overlaps it
        const float wsum = rmw && mr.last ? prm.P.wsum[(int64_t)R.b * Ntok + tok] : 1.f;
        const float tent = (float)(min(y - R.win.x + 1, R.win.x + R.win.z - y) *
                                   min(x - R.win.y + 1, R.win.y + R.win.w - x));
        const int cls = R.cls;
        if (!(ok = warp_wait_all(bO, o_cnt & 1u, abort_flag))) break;
        ++o_cnt;
        tc_fence_after();
        const float inv = 1.f / l;
        if (__any_sync(0xffffffffu, rmw && !mr.first)) {
          int wok = 1;
          if (lane == 0) {
            const uint64_t t0 = global_ns();
            for (int c = 0; c < cls && wok; ++c) {
              // completions class c of this (element, head) needs: 8 warps per unit
              const unsigned target = 8u * (unsigned)prm.P.nclass[R.b * 4 + c];
              const unsigned* ctr = prm.counters + kWsClassDone + bh * 4 + c;
              uint32_t it = 0;
              for (;;) {
                unsigned v;
                asm volatile("ld.acquire.gpu.global.u32 %0, [%1];"
                             : "=r"(v) : "l"(ctr) : "memory");
                if (v >= target) break;
                if ((++it & 63u) == 0) {
                  if (*(volatile int*)abort_flag) { wok = 0; break; }
                  if (global_ns() - t0 > kWaitNs) {
                    *(volatile int*)abort_flag = 1;
                    atomicExch(&g_tc_error, 1);
                    wok = 0;
                    break;
                  }
                }
                __nanosleep(64);
              }
            }
          }
          wok = __shfl_sync(0xffffffffu, wok, 0);
          __threadfence();
          if (!(ok = wok != 0)) break;
        }
        const float sc = mr.ov ? tent * inv : inv;
        const float winv = 1.f / wsum;
        __nv_bfloat16* dsto = prm.o + ((int64_t)bh * Ntok + tok) * D;
        float* acc = prm.acc + ((int64_t)bh * prm.n_ov + mr.rank) * D;
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t orr[32];
          tmem_ld32(tO + c * 32, orr);
          if (!qvalid) continue;
          float vals[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) vals[i] = __uint_as_float(orr[i]) * sc;
          if (rmw) {
            float* a = acc + c * 32;
            if (!mr.first) {
#pragma unroll
              for (int v = 0; v < 4; ++v) {
                float t[8];
                ld_global_v8f(a + 8 * v, t);
#pragma unroll
                for (int i = 0; i < 8; ++i) vals[8 * v + i] += t[i];
              }
            }
            if (!mr.last) {
#pragma unroll
              for (int v = 0; v < 4; ++v) st_global_v8f(a + 8 * v, vals + 8 * v);
              continue;
            }
#pragma unroll
            for (int i = 0; i < 32; ++i) vals[i] *= winv;
          }
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            uint32_t w[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) w[i] = pack_bf16(vals[16 * h + 2 * i], vals[16 * h + 2 * i + 1]);
            st_global_v8(dsto + c * 32 + h * 16, w);
          }
        }
        // this warp's rows of the unit are complete
        __threadfence();
        __syncwarp();
        if (lane == 0) atomicAdd(prm.counters + kWsClassDone + bh * 4 + cls, 1u);
      }
      tc_fence_before();
      if (lane == 0) mbar_arrive(bar(BAR_REC_EMPTY + slot));
      ++unit_count;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem) : "memory");
  }
}

// One CTA per (window slot, element x head): copies the window's global-KV
// rows that fill whole 128-row tiles, K then V, to the staging area
// [B*H][nw][G][D] (rows past those tiles, and windows past the plan's count,
// are skipped: the attention kernel gathers a partial last tile itself).
template <int D>
__global__ void __launch_bounds__(256) stage_list_kernel(const __nv_bfloat16* __restrict__ k,
                                                         const __nv_bfloat16* __restrict__ v,
                                                         const PlanView P, int H,
                                                         __nv_bfloat16* __restrict__ sk,
                                                         __nv_bfloat16* __restrict__ sv) {
  const int w = blockIdx.x, bh = blockIdx.y, b = bh / H;
  if (w >= P.nwin[b]) return;
  const int64_t wo = (int64_t)b * P.nw + w;
  const int nrow = P.gcount[wo] / 128 * 128;
  const int* gl = P.gidx + wo * P.G;
  const int64_t src0 = (int64_t)bh * P.N, dst0 = ((int64_t)bh * P.nw + w) * P.G;
  constexpr int kChunks = D / 8;               // 16-byte chunks per row
  for (int i = threadIdx.x; i < nrow * kChunks; i += blockDim.x) {
    const int r = i / kChunks, c = i % kChunks;
    const int64_t src = (src0 + gl[r]) * D + c * 8, dst = (dst0 + r) * D + c * 8;
    *reinterpret_cast<uint4*>(sk + dst) = *reinterpret_cast<const uint4*>(k + src);
    *reinterpret_cast<uint4*>(sv + dst) = *reinterpret_cast<const uint4*>(v + src);
  }
}

// One CTA per (128-row tile, element x head): copies the head's bridge
// candidate rows of whole 128-row tiles, K then V, to [B*H][R][D].
template <int D>
__global__ void __launch_bounds__(256) stage_cand_kernel(const __nv_bfloat16* __restrict__ k,
                                                         const __nv_bfloat16* __restrict__ v,
                                                         const int* __restrict__ cand, int R,
                                                         int N, __nv_bfloat16* __restrict__ sk,
                                                         __nv_bfloat16* __restrict__ sv) {
  const int t = blockIdx.x, bh = blockIdx.y;
  const int* cl = cand + (int64_t)bh * R + t * 128;
  const int64_t src0 = (int64_t)bh * N, dst0 = (int64_t)bh * R + t * 128;
  constexpr int kChunks = D / 8;
  for (int i = threadIdx.x; i < 128 * kChunks; i += blockDim.x) {
    const int r = i / kChunks, c = i % kChunks;
    const int64_t src = (src0 + cl[r]) * D + c * 8, dst = (dst0 + r) * D + c * 8;
    *reinterpret_cast<uint4*>(sk + dst) = *reinterpret_cast<const uint4*>(k + src);
    *reinterpret_cast<uint4*>(sv + dst) = *reinterpret_cast<const uint4*>(v + src);
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 2-D bf16 map over [rows, D] with a box of 64 columns x box_rows rows.
cudaError_t make_map(CUtensorMap* m, const void* base, int64_t rows, int box_rows, int D) {
  auto enc = get_encode();
  if (!enc) return cudaErrorNotSupported;
  cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)D * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// 3-D bf16 map over [rows_y, Wg, D] (token-grid rows of all (b, h), grid
// columns, head dims) with a box of 64 dims x bw tokens x bh grid rows.
cudaError_t make_map_grid(CUtensorMap* m, const void* base, int64_t rows_y, int Wg, int D, int bw,
                          int bh) {
  auto enc = get_encode();
  if (!enc) return cudaErrorNotSupported;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)Wg, (cuuint64_t)rows_y};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)Wg * D * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)bw, (cuuint32_t)bh};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

int num_sms() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n;
}

template <bool WINDOW, bool BRIDGE, int D>
cudaError_t launch_tc(const TcMaps& maps, const TcParams& prm, cudaStream_t s) {
  constexpr int kSmemBytes = Geo<D>::kSmemBytes;
  constexpr int kThreads = tc_threads(WINDOW);
  auto fn = attn_tc_kernel<WINDOW, BRIDGE, D>;
  if constexpr (WINDOW) {
    // setmaxnreg.inc waits until the registers it asks for are free, so the
    // split must fit in what the launch allocates (registers per thread,
    // rounded down to the allocation unit of 8, times the block's threads)
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, fn);
    if (e != cudaSuccess) return e;
    if (kThreads * (fa.numRegs / 8 * 8) < 128 * kRegsLow + 256 * kRegsHigh)
      return cudaErrorInvalidConfiguration;
  }
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  const int grid = prm.num_units < num_sms() ? prm.num_units : num_sms();
  fn<<<grid > 0 ? grid : 1, kThreads, kSmemBytes, s>>>(maps, prm);
  return cudaGetLastError();
}

}  // namespace

cudaError_t read_and_clear_tc_error(int* code) {
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return e;
  e = cudaMemcpyFromSymbol(code, g_tc_error, sizeof(int));
  if (e != cudaSuccess) return e;
  const int zero = 0;
  return cudaMemcpyToSymbol(g_tc_error, &zero, sizeof(int));
}

cudaError_t launch_dense_attn_tc(const void* q, const void* k, const void* v, const void* kt,
                                 const void* vt, void* o, int B, int H, int N, int Nk, int T,
                                 int D, float scale, cudaStream_t s) {
  TcMaps m;
  cudaError_t e;
  if ((e = make_map(&m.q, q, (int64_t)B * H * N, 128, D)) != cudaSuccess) return e;
  if ((e = make_map(&m.k, k, (int64_t)B * H * Nk, 128, D)) != cudaSuccess) return e;
  if ((e = make_map(&m.v, v, (int64_t)B * H * Nk, 128, D)) != cudaSuccess) return e;
  if (T > 0) {
    if ((e = make_map(&m.kt, kt, (int64_t)B * H * T, 128, D)) != cudaSuccess) return e;
    if ((e = make_map(&m.vt, vt, (int64_t)B * H * T, 128, D)) != cudaSuccess) return e;
  } else {
    m.kt = m.k;   // never read without text keys
    m.vt = m.v;
  }
  m.qc = m.kp = m.vp = m.kc = m.vc = m.ks = m.vs = m.q;   // window maps: never read in dense mode
  TcParams prm{};
  prm.scale_log2 = scale * 1.4426950408889634f;
  prm.H = H;
  prm.T = T;
  prm.da = DenseArgs{B, H, N, Nk, (N + 255) / 256};
  prm.num_units = B * H * prm.da.units_per_head;
  prm.o = static_cast<__nv_bfloat16*>(o);
  if (D == 64) return launch_tc<false, false, 64>(m, prm, s);
  return launch_tc<false, false, 128>(m, prm, s);
}

int64_t window_ws_bytes(const PlanLayout& L, int H, int D) {
  return window_ws_header_bytes(L.B, H) + L.B * H * L.n_ov * D * 4;
}

int64_t window_stage_bytes(const PlanLayout& L, int H, int D) {
  return 2 * L.B * H * L.nw * L.G * D * 2;
}

cudaError_t launch_window_attn_tc(const void* q, const void* k, const void* v, const void* kt,
                                  const void* vt, int T, const int* cand, int R,
                                  const PlanLayout& L, const void* plan, void* o, void* ws,
                                  bool staged, int H, int D, float scale, cudaStream_t s) {
  TcMaps m;
  cudaError_t e;
  const int64_t rows = L.B * H * L.N, rows_y = L.B * H * L.Hg;
  const int Wg = (int)L.Wg;
  if ((e = make_map(&m.q, q, rows, 1, D)) != cudaSuccess) return e;
  if ((e = make_map_grid(&m.qc, q, rows_y, Wg, D, kCW, kCH)) != cudaSuccess) return e;
  if ((e = make_map_grid(&m.kp, k, rows_y, Wg, D, kPW, kPH)) != cudaSuccess) return e;
  if ((e = make_map_grid(&m.vp, v, rows_y, Wg, D, kPW, kPH)) != cudaSuccess) return e;
  if ((e = make_map_grid(&m.kc, k, rows_y, Wg, D, kCW, kCH)) != cudaSuccess) return e;
  if ((e = make_map_grid(&m.vc, v, rows_y, Wg, D, kCW, kCH)) != cudaSuccess) return e;
  m.k = m.kp;   // partial global-KV tiles are copied with cp.async: no row map
  m.v = m.vp;
  // whole global-KV tiles: staged rows after the workspace, [B*H*nw*G, D]
  // (plan lists) or [B*H*R, D] (bridge candidates)
  const int64_t nstage = cand ? L.B * H * R : L.B * H * L.nw * L.G;
  __nv_bfloat16* sk = nullptr;
  __nv_bfloat16* sv = nullptr;
  if (staged && nstage > 0 && nstage < (int64_t(1) << 31)) {
    sk = reinterpret_cast<__nv_bfloat16*>(static_cast<char*>(ws) + window_ws_bytes(L, H, D));
    sv = sk + nstage * D;
    if ((e = make_map(&m.ks, sk, nstage, 128, D)) != cudaSuccess) return e;
    if ((e = make_map(&m.vs, sv, nstage, 128, D)) != cudaSuccess) return e;
  } else {
    staged = false;
    m.ks = m.vs = m.q;   // never read
  }
  if (T > 0) {
    if ((e = make_map(&m.kt, kt, L.B * H * T, 128, D)) != cudaSuccess) return e;
    if ((e = make_map(&m.vt, vt, L.B * H * T, 128, D)) != cudaSuccess) return e;
  } else {
    m.kt = m.q;   // never read without text keys
    m.vt = m.q;
  }
  TcParams prm{};
  prm.scale_log2 = scale * 1.4426950408889634f;
  prm.H = H;
  prm.T = T;
  prm.P = plan_view(L, const_cast<void*>(plan));
  prm.cand = cand;
  prm.R = R;
  prm.num_units = (int)(L.nitem_max * L.B * H);
  prm.o = static_cast<__nv_bfloat16*>(o);
  prm.k = static_cast<const __nv_bfloat16*>(k);
  prm.v = static_cast<const __nv_bfloat16*>(v);
  prm.counters = static_cast<unsigned*>(ws);
  const int64_t hdr = window_ws_header_bytes(L.B, H);
  prm.acc = reinterpret_cast<float*>(static_cast<char*>(ws) + hdr);
  prm.nx2 = (int)L.nx2;
  prm.n_ov = L.n_ov;
  prm.staged = staged ? 1 : 0;
  // unit counter and class completion counters start at zero
  if ((e = cudaMemsetAsync(ws, 0, (size_t)hdr, s)) != cudaSuccess) return e;
  if (staged) {
    const auto* kb = static_cast<const __nv_bfloat16*>(k);
    const auto* vb = static_cast<const __nv_bfloat16*>(v);
    if (cand) {
      const dim3 grid((unsigned)(R / 128), (unsigned)(L.B * H));
      const int N = (int)L.N;
      if (D == 64) stage_cand_kernel<64><<<grid, 256, 0, s>>>(kb, vb, cand, R, N, sk, sv);
      else stage_cand_kernel<128><<<grid, 256, 0, s>>>(kb, vb, cand, R, N, sk, sv);
    } else {
      const dim3 grid((unsigned)L.nw, (unsigned)(L.B * H));
      if (D == 64) stage_list_kernel<64><<<grid, 256, 0, s>>>(kb, vb, prm.P, H, sk, sv);
      else stage_list_kernel<128><<<grid, 256, 0, s>>>(kb, vb, prm.P, H, sk, sv);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  if (D == 64) {
    if (cand) return launch_tc<true, true, 64>(m, prm, s);
    return launch_tc<true, false, 64>(m, prm, s);
  }
  if (cand) return launch_tc<true, true, 128>(m, prm, s);
  return launch_tc<true, false, 128>(m, prm, s);
}

}  // namespace area
