// ptx.cuh -- thin inline-PTX wrappers for sm_100a: mbarriers with bounded
// waits, TMA bulk copies, and the tcgen05 (5th-generation tensor core / TMEM)
// instructions the ternary kernels use.  Nothing here is specific to the
// ternary method.
#pragma once
#include <cstdint>
#include <cuda.h>

namespace tern {

// Bits of the per-device status word.  Kernels OR bits into it (through the
// pointer they are given) instead of trapping; the host reads and clears it.
constexpr unsigned kStatusTimeout = 1u;
// A kernel found its launch configuration inconsistent with its arguments
// (a defect of the host code, never of the caller's data); it computed nothing.
constexpr unsigned kStatusLaunchConfig = 2u;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ bool elect_one() {
  uint32_t pred = 0;
  asm volatile(
      "{\n\t.reg .pred p;\n\t.reg .b32 r;\n\t"
      "elect.sync r|p, 0xffffffff;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(pred));
  return pred != 0;
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
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

// Same test with acquire semantics at cluster scope, for barriers that
// threads of the other CTA of a cluster arrive on.
__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Waits for the phase with the given parity to complete, for at most about
// limit_ns of wall time.  On expiry it records kStatusTimeout in *status and
// returns false; it never traps and never spins forever.  The limit is
// counted in SM clock cycles (cheap to read) at 2 cycles per ns, so it is a
// wall-time bound of limit_ns * 2 / f_sm: about limit_ns at the B200's
// 1.9-2.0 GHz boost and longer at lower clocks; the clock is read only every
// 64 polls so that waiting warps stay off the issue slots of working ones.
template <bool kCluster = false>
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, uint64_t limit_ns,
                                          unsigned int* status) {
  auto poll = [&]() { return kCluster ? mbar_try_wait_cluster(bar, parity) : mbar_try_wait(bar, parity); };
  if (poll()) return true;
  const long long t0 = clock64();
  const long long limit_cycles = (long long)(limit_ns * 2ull);
#pragma unroll 1
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 64; ++i)
      if (poll()) return true;
    if (clock64() - t0 > limit_cycles) {
      atomicOr(status, kStatusTimeout);
      return false;
    }
  }
}

// Both phases, as mbar_wait each: the first two polls go out back to back,
// so when both phases are already complete (the usual case) the wait costs
// one poll's latency instead of two.
__device__ __forceinline__ bool mbar_wait_both(uint32_t bar0, uint32_t parity0, uint32_t bar1, uint32_t parity1,
                                               uint64_t limit_ns, unsigned int* status) {
  const bool d0 = mbar_try_wait(bar0, parity0);
  const bool d1 = mbar_try_wait(bar1, parity1);
  if (d0 && d1) return true;
  return (d0 || mbar_wait(bar0, parity0, limit_ns, status)) && (d1 || mbar_wait(bar1, parity1, limit_ns, status));
}

// Programmatic dependent launch.  Our kernels are launched with it allowed,
// so a grid may start while the previous kernel of its stream still runs:
// every kernel calls pdl_wait() before it touches global memory (it returns
// once the previous grid has finished and its writes are visible; at once
// when there is none), then pdl_trigger() lets the next kernel be scheduled.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Asks L2 to fetch [p, p + bytes) (16-byte aligned, a multiple of 16 bytes);
// a hint with no result and no ordering.
__device__ __forceinline__ void prefetch_l2_bulk(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// Asks for the 128-byte line holding `p` to be brought into L2 (no register
// result, no ordering).
__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// ------------------------------------------------------------- TMA copies
// Untiled bulk copy global -> shared, completing bytes on an mbarrier.
// Both addresses 16-byte aligned, size a multiple of 16.
__device__ __forceinline__ void tma_load_bulk(uint32_t dst, const void* src, uint32_t bytes,
                                              uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

// Tiled 2-D tensor copy global -> shared (box and swizzle from the map).
// c0 is the innermost coordinate in elements and must be 16-byte aligned.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int32_t c0,
                                            int32_t c1, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(bar)
      : "memory");
}

// Tiled 3-D tensor copy global -> shared (box and swizzle from the map).
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, int32_t c0, int32_t c1,
                                            int32_t c2, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(
          dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ------------------------------------------------------------------ tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]^T, kind::f16 (bf16 inputs, fp32 accumulate).
__device__ __forceinline__ void mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive (once) on an mbarrier when every tcgen05 op this thread issued so far is done.
__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}

__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Each thread of the warp writes 16 / 32 consecutive 32-bit columns of its own lane.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
      : "memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]),
      "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]),
      "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
}

// Each thread of the warp reads 16 consecutive 32-bit columns of its own lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
        "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]),
        "=r"(v[14]), "=r"(v[15])
      : "r"(taddr)
      : "memory");
}

// Each thread of the warp reads 32 consecutive 32-bit columns of its own lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
        "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]),
        "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]),
        "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]),
        "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
      : "r"(taddr)
      : "memory");
}

// ------------------------------------------------------------ clusters
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
__device__ __forceinline__ uint32_t nclusters_x() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
  return r;
}
// Address of the same shared-memory variable in CTA `cta` of this cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t cta) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(cta));
  return r;
}
// Arrive on an mbarrier given by a shared::cluster address (possibly in the
// other CTA of the cluster).  The default (CTA-scope release) semantics are
// enough for what crosses the pair here: TMEM and shared-memory operands that
// the arriving thread has already waited on (tcgen05.wait, mbarrier), read by
// tcgen05 operations of the other CTA.  A cluster-scope release costs about a
// thousand cycles per arrival under load, which would throttle the pipeline.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
// 32-bit load from shared memory of any CTA of the cluster (address from mapa).
__device__ __forceinline__ float ld_shared_cluster_f32(uint32_t cluster_addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(cluster_addr) : "memory");
  return v;
}
// All threads of every CTA of the cluster, ordering nothing: for a final
// rendezvous after which no shared memory of another CTA is read.
__device__ __forceinline__ void cluster_sync_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;\n\tbarrier.cluster.wait.aligned;" ::: "memory");
}
// All threads of every CTA of the cluster.
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" :::
                   "memory");
}

// 2-SM (cta_group::2) forms: the CTA pair shares one MMA; each CTA holds half
// of A (its 128 rows), half of B (N/2 rows) and its 128 rows of D.
__device__ __forceinline__ void tmem_alloc_2sm(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_2sm() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_2sm(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
// Commits issued, like mma_stage, by the lane elect.sync picks in a
// converged warp (all 32 lanes call them): the mbarrier gets one arrival when
// every tcgen05 op that lane issued so far is done.  The 2-SM multicast form
// arrives at the same shared-memory offset in every CTA of `cta_mask`.
__device__ __forceinline__ void mma_commit_elected(uint32_t bar) {
  asm volatile(
      "{\n\t.reg .pred p;\n\telect.sync _|p, 0xffffffff;\n\t"
      "@p tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(bar)
      : "memory");
}
__device__ __forceinline__ void mma_commit_2sm_multicast_elected(uint32_t bar, uint16_t cta_mask) {
  asm volatile(
      "{\n\t.reg .pred p;\n\telect.sync _|p, 0xffffffff;\n\t"
      "@p tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;\n\t}"
      ::"r"(bar), "h"(cta_mask)
      : "memory");
}
__device__ __forceinline__ void mma_commit_2sm_elected(uint32_t bar) {
  asm volatile(
      "{\n\t.reg .pred p;\n\telect.sync _|p, 0xffffffff;\n\t"
      "@p tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(bar)
      : "memory");
}

// One 128-k stage of the tile kernels issued at once: NMMA k16 MMAs (8, or 4
// for a 64-k tail) followed by two commits, all from the lane that elect.sync
// picks in a converged warp (later commits covering these MMAs go through the
// *_elected forms below, called by the same converged warp, so they come from
// that lane too).  Every lane computes the same operands, so they stay
// warp-uniform; issuing the same instructions from a single-lane branch with
// per-MMA descriptor arithmetic was measured to take several times the MMA's
// own duration at N = 64, and a lane-0 predicate instead of elect.sync ~13 %
// longer per tile at N = 64.
//   d        accumulator TMEM address
//   a        TMEM column address of k16 step 0 of A; step j reads a + 8 j
//   desc     shared-memory descriptor of B's step 0; step j adds 32 bytes
//            (2 in the address field) inside a 64-k chunk, and `chunk2` (the
//            second chunk's byte offset >> 4) for j >= 4
//   acc      0 for the first stage of a tile (D = A B), else D += A B
//   bar0/1   mbarriers the commits arrive on (PAIR: in both CTAs of the pair)
#define TERN_STAGE_PROLOGUE                                            \
  "{\n\t.reg .pred p, q, t;\n\t"                                      \
  ".reg .b64 e1, e2, e3, e4, e5, e6, e7;\n\t"                         \
  ".reg .b32 a1, a2, a3, a4, a5, a6, a7;\n\t"                         \
  "elect.sync _|p, 0xffffffff;\n\t"                                   \
  "setp.ne.b32 q, %4, 0;\n\t"                                         \
  "setp.eq.b32 t, 0, 0;\n\t"                                          \
  "add.s64 e1, %2, 2;\n\t add.s64 e2, %2, 4;\n\t add.s64 e3, %2, 6;\n\t" \
  "add.s64 e4, %2, %7;\n\t add.s64 e5, e4, 2;\n\t"                    \
  "add.s64 e6, e4, 4;\n\t add.s64 e7, e4, 6;\n\t"                     \
  "add.u32 a1, %1, 8;\n\t add.u32 a2, %1, 16;\n\t add.u32 a3, %1, 24;\n\t" \
  "add.u32 a4, %1, 32;\n\t add.u32 a5, %1, 40;\n\t"                   \
  "add.u32 a6, %1, 48;\n\t add.u32 a7, %1, 56;\n\t"
#define TERN_STAGE_MMA(G, A, E, P) "@p tcgen05.mma.cta_group::" #G ".kind::f16 [%0], [" A "], " E ", %3, " P ";\n\t"
#define TERN_STAGE_LO(G) \
  TERN_STAGE_MMA(G, "%1", "%2", "q") TERN_STAGE_MMA(G, "a1", "e1", "t") \
  TERN_STAGE_MMA(G, "a2", "e2", "t") TERN_STAGE_MMA(G, "a3", "e3", "t")
#define TERN_STAGE_HI(G) \
  TERN_STAGE_MMA(G, "a4", "e4", "t") TERN_STAGE_MMA(G, "a5", "e5", "t") \
  TERN_STAGE_MMA(G, "a6", "e6", "t") TERN_STAGE_MMA(G, "a7", "e7", "t")
#define TERN_COMMIT1(BAR) "@p tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [" BAR "];\n\t"
#define TERN_COMMIT2(BAR) \
  "@p tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [" BAR "], %8;\n\t"

template <int NMMA, bool PAIR>
__device__ __forceinline__ void mma_stage(uint32_t d, uint32_t a, uint64_t desc, uint32_t idesc, uint32_t acc,
                                          uint32_t bar0, uint32_t bar1, uint64_t chunk2) {
  static_assert(NMMA == 4 || NMMA == 8, "a stage is one or two 64-k chunks");
  const uint16_t both = 0x3;  // commit multicast: both CTAs of the pair
  if constexpr (!PAIR && NMMA == 8)
    asm volatile(TERN_STAGE_PROLOGUE TERN_STAGE_LO(1) TERN_STAGE_HI(1) TERN_COMMIT1("%5") TERN_COMMIT1("%6") "}"
                 ::"r"(d), "r"(a), "l"(desc), "r"(idesc), "r"(acc), "r"(bar0), "r"(bar1), "l"(chunk2), "h"(both)
                 : "memory");
  else if constexpr (!PAIR)
    asm volatile(TERN_STAGE_PROLOGUE TERN_STAGE_LO(1) TERN_COMMIT1("%5") TERN_COMMIT1("%6") "}"
                 ::"r"(d), "r"(a), "l"(desc), "r"(idesc), "r"(acc), "r"(bar0), "r"(bar1), "l"(chunk2), "h"(both)
                 : "memory");
  else if constexpr (NMMA == 8)
    asm volatile(TERN_STAGE_PROLOGUE TERN_STAGE_LO(2) TERN_STAGE_HI(2) TERN_COMMIT2("%5") TERN_COMMIT2("%6") "}"
                 ::"r"(d), "r"(a), "l"(desc), "r"(idesc), "r"(acc), "r"(bar0), "r"(bar1), "l"(chunk2), "h"(both)
                 : "memory");
  else
    asm volatile(TERN_STAGE_PROLOGUE TERN_STAGE_LO(2) TERN_COMMIT2("%5") TERN_COMMIT2("%6") "}"
                 ::"r"(d), "r"(a), "l"(desc), "r"(idesc), "r"(acc), "r"(bar0), "r"(bar1), "l"(chunk2), "h"(both)
                 : "memory");
}
// The first 128 k of a longer stage: eight MMAs like mma_stage<8>, no
// commit (the commits after the stage's last block cover them: a commit
// tracks every tcgen05 op its thread issued before it, and elect.sync picks
// the same lane of the converged warp each time).
template <bool PAIR>
__device__ __forceinline__ void mma_stage_open(uint32_t d, uint32_t a, uint64_t desc, uint32_t idesc, uint32_t acc,
                                               uint64_t chunk2) {
  if constexpr (!PAIR)
    asm volatile(TERN_STAGE_PROLOGUE TERN_STAGE_LO(1) TERN_STAGE_HI(1) "}"
                 ::"r"(d), "r"(a), "l"(desc), "r"(idesc), "r"(acc), "r"(0u), "r"(0u), "l"(chunk2)
                 : "memory");
  else
    asm volatile(TERN_STAGE_PROLOGUE TERN_STAGE_LO(2) TERN_STAGE_HI(2) "}"
                 ::"r"(d), "r"(a), "l"(desc), "r"(idesc), "r"(acc), "r"(0u), "r"(0u), "l"(chunk2)
                 : "memory");
}
#undef TERN_STAGE_PROLOGUE
#undef TERN_STAGE_MMA
#undef TERN_STAGE_LO
#undef TERN_STAGE_HI
#undef TERN_COMMIT1
#undef TERN_COMMIT2

// Named barrier over a subset of the CTA's warps that also ANDs a predicate
// across them (every participating thread gets the same answer).
__device__ __forceinline__ bool named_barrier_and(uint32_t id, uint32_t nthreads, bool pred) {
  uint32_t out;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %3, 0;\n\t"
      "bar.red.and.pred q, %1, %2, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(out)
      : "r"(id), "r"(nthreads), "r"(uint32_t(pred))
      : "memory");
  return out != 0;
}

// Named barrier over a subset of the CTA's warps.
__device__ __forceinline__ void named_barrier_sync(uint32_t id, uint32_t nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

}  // namespace tern
