// sm100_ptx.cuh -- thin inline-PTX wrappers for the Blackwell (sm_100a) features the
// tensor-core retention kernel uses: mbarriers with bounded waits, TMA tile loads (no
// multicast), tcgen05 TMEM allocation, MMA, commit, TMEM loads/stores and fences, and the
// shared-memory matrix descriptors of the 128-byte-swizzled canonical layouts.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace retnet {
namespace sm100 {

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---- mbarrier ------------------------------------------------------------------------------

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
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

// Count of bounded waits that gave up in kernels of the including file (a kernel that hits
// one stops its work, releases what it holds and returns; the host reads and clears it).
// Programmatic dependent launch: let the grid launched after this one (with the
// programmatic-serialization attribute) start; and, in that grid, wait until the grid before
// it has completed and its memory writes are visible.
__device__ __forceinline__ void griddep_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Non-blocking probe of an mbarrier phase.
__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

static __device__ unsigned int g_wait_timeouts = 0;
// Budget, in SM clock cycles, of a wait for another role's progress (about 2 s by default).  A
// host-side testing aid may lower it so that waits give up; waits for work this thread already
// issued (TMA loads, MMAs) always take kDrainBudget, so a kernel that gave up never leaves with
// copies or products in flight.
constexpr long long kDrainBudget = 4000000000LL;
// In constant memory: every bounded wait (and the MMA issuer's polling loop) reads it, and a
// global-memory read there put a memory latency into the wait for an mbarrier phase.  The host
// changes it only between launches (retnet_debug_set_wait_budget synchronises first).
static __constant__ long long g_wait_budget = kDrainBudget;
// Threads that rounded a value outside the fp16 range (magnitude >= 65520 becomes inf, or NaN)
// when forming a tensor-core operand: bf16 inputs span a far wider range than fp16 operands.
static __device__ unsigned int g_fp16_overflows = 0;

// One report per thread: mx is the largest magnitude the thread rounded to fp16 (NaN-safe).
__device__ __forceinline__ void report_fp16_range(float mx) {
  if (!(mx < 65520.f)) atomicAdd(&g_fp16_overflows, 1u);
}
// Largest magnitude so far, NaN sticky (max.NaN propagates a NaN where fmaxf would drop it).
__device__ __forceinline__ float absmax(float m, float x) {
  float r;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(m), "f"(fabsf(x)));
  return r;
}

// ---- thread-block clusters: distributed shared memory, remote mbarrier arrivals --------------

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// All threads of all CTAs of the cluster (the CTAs of a cluster are co-scheduled, so every one
// of them reaches it: used once after set-up and once before exit, never inside a loop).
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Address of the same shared-memory location in CTA `rank` of this cluster.
__device__ __forceinline__ uint32_t map_shared_rank(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
__device__ __forceinline__ void st_cluster_v2(uint32_t addr, float a, float b) {
  asm volatile("st.shared::cluster.v2.f32 [%0], {%1, %2};" ::"r"(addr), "f"(a), "f"(b) : "memory");
}
// Asynchronous 8-byte store into another CTA's shared memory that completes 8 bytes of
// transaction count on that CTA's mbarrier (both addresses from map_shared_rank): the data is
// visible to whoever observes the phase it completes, with no fence on the sending side.
__device__ __forceinline__ void st_async_v2(uint32_t remote_addr, float a, float b, uint32_t remote_bar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v2.f32 [%0], {%1, %2}, [%3];" ::"r"(remote_addr),
               "f"(a), "f"(b), "r"(remote_bar)
               : "memory");
}
// Arrive on an mbarrier of another CTA of the cluster; release at cluster scope orders this
// thread's earlier writes (to that CTA's shared memory) before the arrival.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t remote_bar) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(remote_bar) : "memory");
}
// Bounded wait on a local mbarrier whose arrivals come from the cluster (acquire at cluster scope).
__device__ __forceinline__ bool mbar_wait_cluster(uint32_t bar, uint32_t parity, long long budget = -1) {
  auto probe = [&]() -> bool {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
  };
  if (probe()) return true;
  if (budget < 0) budget = g_wait_budget;
  const long long t0 = clock64();
  while (!probe()) {
    if (clock64() - t0 > budget) {
      atomicAdd(&g_wait_timeouts, 1u);
      return false;
    }
  }
  return true;
}


// Waits for the phase with the given parity to complete, for at most `budget` SM clock
// cycles (default: the pipeline budget g_wait_budget).  Returns false (and counts a timeout)
// if it gave up.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, long long budget = -1) {
  if (mbar_try_wait(bar, parity)) return true;
  if (budget < 0) budget = g_wait_budget;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > budget) {
      atomicAdd(&g_wait_timeouts, 1u);
      return false;
    }
  }
  return true;
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void named_bar_sync(uint32_t id, uint32_t threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// ---- TMA (tile mode, no multicast) -----------------------------------------------------------

__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap* map, uint32_t bar, int c0, int c1, int c2,
                                            int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, %5}], "
      "[%6];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ---- tcgen05: TMEM allocation -----------------------------------------------------------------

__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// ---- tcgen05: MMA ----------------------------------------------------------------------------

// D[tmem] (+)= A[smem] * B[smem], kind::f16 (fp16 or bf16 operands, fp32 accumulate).
__device__ __forceinline__ void mma_f16_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                           uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive once on `bar` when every tcgen05 operation this thread issued before has completed.
__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

// Instruction descriptor of kind::f16 with fp16 A and B, fp32 D; a_mn / b_mn select
// MN-major (1) or K-major (0) operands.
__host__ __device__ constexpr uint32_t idesc_f16_f32(int M, int N, int a_mn, int b_mn) {
  return (1u << 4)                                  // D format: f32
         | (0u << 7) | (0u << 10)                   // A, B format: f16
         | (static_cast<uint32_t>(a_mn) << 15) | (static_cast<uint32_t>(b_mn) << 16) |
         (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

// Shared-memory matrix descriptor, 128-byte swizzle, sm_100 version field.
//   K-major:  rows of 128 B (64 fp16 along K), 8-row atoms every `sbo` bytes; `lbo` unused (16).
//   MN-major: 128-B rows along MN (64 fp16), one row per K index, 8-row atoms every `sbo`
//             bytes along K, 64-element MN blocks every `lbo` bytes.
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  return static_cast<uint64_t>((addr >> 4) & 0x3FFFu) | (static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16) |
         (static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

// ---- tcgen05: TMEM <-> registers --------------------------------------------------------------

// TMEM loads, 32 lanes x 32 bits: thread i of the warp reads lane (warp base + i), consecutive
// columns into consecutive registers.  tcgen05.ld completes asynchronously, and an inline-asm
// output is taken by the compiler as written when its statement ends; so every load here is
// issued together with its tcgen05.wait::ld in ONE asm statement, which leaves the compiler no
// point at which it could read, move or spill a destination register before the data lands.

// 16 columns.
__device__ __forceinline__ void tmem_ld_wait(uint32_t taddr, uint32_t (&r)[1][16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15}, [%16]; tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0][0]), "=r"(r[0][1]), "=r"(r[0][2]), "=r"(r[0][3]), "=r"(r[0][4]), "=r"(r[0][5]), "=r"(r[0][6]),
        "=r"(r[0][7]), "=r"(r[0][8]), "=r"(r[0][9]), "=r"(r[0][10]), "=r"(r[0][11]), "=r"(r[0][12]),
        "=r"(r[0][13]), "=r"(r[0][14]), "=r"(r[0][15])
      : "r"(taddr)
      : "memory");
}

// 16 columns from each of two addresses, one wait.
__device__ __forceinline__ void tmem_ld_wait(uint32_t ta, uint32_t (&ra)[1][16], uint32_t tb, uint32_t (&rb)[1][16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15}, [%32]; tcgen05.ld.sync.aligned.32x32b.x16.b32 {%16, %17, %18, %19, "
      "%20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%33]; "
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(ra[0][0]), "=r"(ra[0][1]), "=r"(ra[0][2]), "=r"(ra[0][3]), "=r"(ra[0][4]), "=r"(ra[0][5]),
        "=r"(ra[0][6]), "=r"(ra[0][7]), "=r"(ra[0][8]), "=r"(ra[0][9]), "=r"(ra[0][10]), "=r"(ra[0][11]),
        "=r"(ra[0][12]), "=r"(ra[0][13]), "=r"(ra[0][14]), "=r"(ra[0][15]), "=r"(rb[0][0]), "=r"(rb[0][1]),
        "=r"(rb[0][2]), "=r"(rb[0][3]), "=r"(rb[0][4]), "=r"(rb[0][5]), "=r"(rb[0][6]), "=r"(rb[0][7]),
        "=r"(rb[0][8]), "=r"(rb[0][9]), "=r"(rb[0][10]), "=r"(rb[0][11]), "=r"(rb[0][12]), "=r"(rb[0][13]),
        "=r"(rb[0][14]), "=r"(rb[0][15])
      : "r"(ta), "r"(tb)
      : "memory");
}

// 32 columns.
__device__ __forceinline__ void tmem_ld_wait(uint32_t taddr, uint32_t (&r)[2][16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, "
      "%30, %31}, [%32]; tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0][0]), "=r"(r[0][1]), "=r"(r[0][2]), "=r"(r[0][3]), "=r"(r[0][4]), "=r"(r[0][5]), "=r"(r[0][6]),
        "=r"(r[0][7]), "=r"(r[0][8]), "=r"(r[0][9]), "=r"(r[0][10]), "=r"(r[0][11]), "=r"(r[0][12]),
        "=r"(r[0][13]), "=r"(r[0][14]), "=r"(r[0][15]), "=r"(r[1][0]), "=r"(r[1][1]), "=r"(r[1][2]),
        "=r"(r[1][3]), "=r"(r[1][4]), "=r"(r[1][5]), "=r"(r[1][6]), "=r"(r[1][7]), "=r"(r[1][8]), "=r"(r[1][9]),
        "=r"(r[1][10]), "=r"(r[1][11]), "=r"(r[1][12]), "=r"(r[1][13]), "=r"(r[1][14]), "=r"(r[1][15])
      : "r"(taddr)
      : "memory");
}

// M = 64 accumulator tiles keep their rows in lanes 0-15 of each lane quarter.  This load
// gives every thread of the warp 32 columns of one of those rows: thread i < 16 row i, columns
// [c, c + 32); thread i + 16 row i, columns [c + OFF, c + OFF + 32) (c = the address's column).
template <int OFF>
__device__ __forceinline__ void tmem_ld16x2_wait(uint32_t taddr, uint32_t (&r)[2][16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.16x32bx2.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32], %33; tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0][0]), "=r"(r[0][1]), "=r"(r[0][2]), "=r"(r[0][3]), "=r"(r[0][4]), "=r"(r[0][5]), "=r"(r[0][6]), "=r"(r[0][7]), "=r"(r[0][8]), "=r"(r[0][9]), "=r"(r[0][10]), "=r"(r[0][11]), "=r"(r[0][12]), "=r"(r[0][13]), "=r"(r[0][14]), "=r"(r[0][15]), "=r"(r[1][0]), "=r"(r[1][1]), "=r"(r[1][2]), "=r"(r[1][3]), "=r"(r[1][4]), "=r"(r[1][5]), "=r"(r[1][6]), "=r"(r[1][7]), "=r"(r[1][8]), "=r"(r[1][9]), "=r"(r[1][10]), "=r"(r[1][11]), "=r"(r[1][12]), "=r"(r[1][13]), "=r"(r[1][14]), "=r"(r[1][15])
      : "r"(taddr), "n"(OFF)
      : "memory");
}

// The same from two addresses (two accumulators of the same layout), one wait.
template <int OFF>
__device__ __forceinline__ void tmem_ld16x2_wait(uint32_t ta, uint32_t (&ra)[2][16], uint32_t tb, uint32_t (&rb)[2][16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.16x32bx2.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%64], %66; "
      "tcgen05.ld.sync.aligned.16x32bx2.x32.b32 {%32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, %48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63}, [%65], %66; tcgen05.wait::ld.sync.aligned;"
      : "=r"(ra[0][0]), "=r"(ra[0][1]), "=r"(ra[0][2]), "=r"(ra[0][3]), "=r"(ra[0][4]), "=r"(ra[0][5]), "=r"(ra[0][6]), "=r"(ra[0][7]), "=r"(ra[0][8]), "=r"(ra[0][9]), "=r"(ra[0][10]), "=r"(ra[0][11]), "=r"(ra[0][12]), "=r"(ra[0][13]), "=r"(ra[0][14]), "=r"(ra[0][15]), "=r"(ra[1][0]), "=r"(ra[1][1]), "=r"(ra[1][2]), "=r"(ra[1][3]), "=r"(ra[1][4]), "=r"(ra[1][5]), "=r"(ra[1][6]), "=r"(ra[1][7]), "=r"(ra[1][8]), "=r"(ra[1][9]), "=r"(ra[1][10]), "=r"(ra[1][11]), "=r"(ra[1][12]), "=r"(ra[1][13]), "=r"(ra[1][14]), "=r"(ra[1][15]), "=r"(rb[0][0]), "=r"(rb[0][1]), "=r"(rb[0][2]), "=r"(rb[0][3]), "=r"(rb[0][4]), "=r"(rb[0][5]), "=r"(rb[0][6]), "=r"(rb[0][7]), "=r"(rb[0][8]), "=r"(rb[0][9]), "=r"(rb[0][10]), "=r"(rb[0][11]), "=r"(rb[0][12]), "=r"(rb[0][13]), "=r"(rb[0][14]), "=r"(rb[0][15]), "=r"(rb[1][0]), "=r"(rb[1][1]), "=r"(rb[1][2]), "=r"(rb[1][3]), "=r"(rb[1][4]), "=r"(rb[1][5]), "=r"(rb[1][6]), "=r"(rb[1][7]), "=r"(rb[1][8]), "=r"(rb[1][9]), "=r"(rb[1][10]), "=r"(rb[1][11]), "=r"(rb[1][12]), "=r"(rb[1][13]), "=r"(rb[1][14]), "=r"(rb[1][15])
      : "r"(ta), "r"(tb), "n"(OFF)
      : "memory");
}

// 64 columns.
__device__ __forceinline__ void tmem_ld_wait(uint32_t taddr, uint32_t (&r)[4][16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x64.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, "
      "%30, %31, %32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, "
      "%48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63}, [%64]; "
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0][0]), "=r"(r[0][1]), "=r"(r[0][2]), "=r"(r[0][3]), "=r"(r[0][4]), "=r"(r[0][5]), "=r"(r[0][6]),
        "=r"(r[0][7]), "=r"(r[0][8]), "=r"(r[0][9]), "=r"(r[0][10]), "=r"(r[0][11]), "=r"(r[0][12]),
        "=r"(r[0][13]), "=r"(r[0][14]), "=r"(r[0][15]), "=r"(r[1][0]), "=r"(r[1][1]), "=r"(r[1][2]),
        "=r"(r[1][3]), "=r"(r[1][4]), "=r"(r[1][5]), "=r"(r[1][6]), "=r"(r[1][7]), "=r"(r[1][8]), "=r"(r[1][9]),
        "=r"(r[1][10]), "=r"(r[1][11]), "=r"(r[1][12]), "=r"(r[1][13]), "=r"(r[1][14]), "=r"(r[1][15]),
        "=r"(r[2][0]), "=r"(r[2][1]), "=r"(r[2][2]), "=r"(r[2][3]), "=r"(r[2][4]), "=r"(r[2][5]), "=r"(r[2][6]),
        "=r"(r[2][7]), "=r"(r[2][8]), "=r"(r[2][9]), "=r"(r[2][10]), "=r"(r[2][11]), "=r"(r[2][12]),
        "=r"(r[2][13]), "=r"(r[2][14]), "=r"(r[2][15]), "=r"(r[3][0]), "=r"(r[3][1]), "=r"(r[3][2]),
        "=r"(r[3][3]), "=r"(r[3][4]), "=r"(r[3][5]), "=r"(r[3][6]), "=r"(r[3][7]), "=r"(r[3][8]), "=r"(r[3][9]),
        "=r"(r[3][10]), "=r"(r[3][11]), "=r"(r[3][12]), "=r"(r[3][13]), "=r"(r[3][14]), "=r"(r[3][15])
      : "r"(taddr)
      : "memory");
}

// 32 columns from each of two addresses, one wait.
__device__ __forceinline__ void tmem_ld_wait(uint32_t ta, uint32_t (&ra)[2][16], uint32_t tb, uint32_t (&rb)[2][16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, "
      "%30, %31}, [%64]; tcgen05.ld.sync.aligned.32x32b.x32.b32 {%32, %33, %34, %35, %36, %37, "
      "%38, %39, %40, %41, %42, %43, %44, %45, %46, %47, %48, %49, %50, %51, %52, %53, %54, %55, "
      "%56, %57, %58, %59, %60, %61, %62, %63}, [%65]; tcgen05.wait::ld.sync.aligned;"
      : "=r"(ra[0][0]), "=r"(ra[0][1]), "=r"(ra[0][2]), "=r"(ra[0][3]), "=r"(ra[0][4]), "=r"(ra[0][5]),
        "=r"(ra[0][6]), "=r"(ra[0][7]), "=r"(ra[0][8]), "=r"(ra[0][9]), "=r"(ra[0][10]), "=r"(ra[0][11]),
        "=r"(ra[0][12]), "=r"(ra[0][13]), "=r"(ra[0][14]), "=r"(ra[0][15]), "=r"(ra[1][0]), "=r"(ra[1][1]),
        "=r"(ra[1][2]), "=r"(ra[1][3]), "=r"(ra[1][4]), "=r"(ra[1][5]), "=r"(ra[1][6]), "=r"(ra[1][7]),
        "=r"(ra[1][8]), "=r"(ra[1][9]), "=r"(ra[1][10]), "=r"(ra[1][11]), "=r"(ra[1][12]), "=r"(ra[1][13]),
        "=r"(ra[1][14]), "=r"(ra[1][15]), "=r"(rb[0][0]), "=r"(rb[0][1]), "=r"(rb[0][2]), "=r"(rb[0][3]),
        "=r"(rb[0][4]), "=r"(rb[0][5]), "=r"(rb[0][6]), "=r"(rb[0][7]), "=r"(rb[0][8]), "=r"(rb[0][9]),
        "=r"(rb[0][10]), "=r"(rb[0][11]), "=r"(rb[0][12]), "=r"(rb[0][13]), "=r"(rb[0][14]), "=r"(rb[0][15]),
        "=r"(rb[1][0]), "=r"(rb[1][1]), "=r"(rb[1][2]), "=r"(rb[1][3]), "=r"(rb[1][4]), "=r"(rb[1][5]),
        "=r"(rb[1][6]), "=r"(rb[1][7]), "=r"(rb[1][8]), "=r"(rb[1][9]), "=r"(rb[1][10]), "=r"(rb[1][11]),
        "=r"(rb[1][12]), "=r"(rb[1][13]), "=r"(rb[1][14]), "=r"(rb[1][15])
      : "r"(ta), "r"(tb)
      : "memory");
}

// TMEM store of 32 columns with its wait.
__device__ __forceinline__ void tmem_st_wait(uint32_t taddr, const uint32_t (&r)[2][16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, "
      "%29, %30, %31, %32}; tcgen05.wait::st.sync.aligned;"
      ::"r"(taddr),
        "r"(r[0][0]), "r"(r[0][1]), "r"(r[0][2]), "r"(r[0][3]), "r"(r[0][4]), "r"(r[0][5]), "r"(r[0][6]),
        "r"(r[0][7]), "r"(r[0][8]), "r"(r[0][9]), "r"(r[0][10]), "r"(r[0][11]), "r"(r[0][12]), "r"(r[0][13]),
        "r"(r[0][14]), "r"(r[0][15]), "r"(r[1][0]), "r"(r[1][1]), "r"(r[1][2]), "r"(r[1][3]), "r"(r[1][4]),
        "r"(r[1][5]), "r"(r[1][6]), "r"(r[1][7]), "r"(r[1][8]), "r"(r[1][9]), "r"(r[1][10]), "r"(r[1][11]),
        "r"(r[1][12]), "r"(r[1][13]), "r"(r[1][14]), "r"(r[1][15])
      : "memory");
}

// TMEM store of 64 columns, with its tcgen05.wait::st in the same statement (the source
// registers stay untouched until the store has read them).
__device__ __forceinline__ void tmem_st_wait(uint32_t taddr, const uint32_t (&r)[4][16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x64.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, "
      "%29, %30, %31, %32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, "
      "%47, %48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63, "
      "%64}; tcgen05.wait::st.sync.aligned;"
      ::"r"(taddr),
        "r"(r[0][0]), "r"(r[0][1]), "r"(r[0][2]), "r"(r[0][3]), "r"(r[0][4]), "r"(r[0][5]), "r"(r[0][6]),
        "r"(r[0][7]), "r"(r[0][8]), "r"(r[0][9]), "r"(r[0][10]), "r"(r[0][11]), "r"(r[0][12]), "r"(r[0][13]),
        "r"(r[0][14]), "r"(r[0][15]), "r"(r[1][0]), "r"(r[1][1]), "r"(r[1][2]), "r"(r[1][3]), "r"(r[1][4]),
        "r"(r[1][5]), "r"(r[1][6]), "r"(r[1][7]), "r"(r[1][8]), "r"(r[1][9]), "r"(r[1][10]), "r"(r[1][11]),
        "r"(r[1][12]), "r"(r[1][13]), "r"(r[1][14]), "r"(r[1][15]), "r"(r[2][0]), "r"(r[2][1]), "r"(r[2][2]),
        "r"(r[2][3]), "r"(r[2][4]), "r"(r[2][5]), "r"(r[2][6]), "r"(r[2][7]), "r"(r[2][8]), "r"(r[2][9]),
        "r"(r[2][10]), "r"(r[2][11]), "r"(r[2][12]), "r"(r[2][13]), "r"(r[2][14]), "r"(r[2][15]), "r"(r[3][0]),
        "r"(r[3][1]), "r"(r[3][2]), "r"(r[3][3]), "r"(r[3][4]), "r"(r[3][5]), "r"(r[3][6]), "r"(r[3][7]),
        "r"(r[3][8]), "r"(r[3][9]), "r"(r[3][10]), "r"(r[3][11]), "r"(r[3][12]), "r"(r[3][13]), "r"(r[3][14]),
        "r"(r[3][15])
      : "memory");
}

// ---- small helpers -------------------------------------------------------------------------

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// (a, b) as two fp16 pairs: hi = fp16(x) and lo = fp16(x - hi) (the difference is exact in fp32),
// so hi + lo carries about 22 significant bits of x.
__device__ __forceinline__ void split_f16x2(float a, float b, uint32_t& hi, uint32_t& lo) {
  const __half2 h = __floats2half2_rn(a, b);
  const float2 hf = __half22float2(h);
  const __half2 l = __floats2half2_rn(a - hf.x, b - hf.y);
  hi = *reinterpret_cast<const uint32_t*>(&h);
  lo = *reinterpret_cast<const uint32_t*>(&l);
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

__device__ __forceinline__ void ld_shared_v4(uint32_t addr, uint32_t& a, uint32_t& b, uint32_t& c, uint32_t& d) {
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(a), "=r"(b), "=r"(c), "=r"(d) : "r"(addr) : "memory");
}

// Byte offset of 16-byte chunk `chunk` of row `row` in a 128-byte-swizzled tile of 128-B rows.
__device__ __forceinline__ uint32_t sw128(uint32_t row, uint32_t chunk) {
  return row * 128u + (((chunk ^ (row & 7u)) & 7u) << 4);
}

}  // namespace sm100
}  // namespace retnet
