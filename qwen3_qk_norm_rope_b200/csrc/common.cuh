// common.cuh - PTX wrappers (mbarrier, TMA, tcgen05, bf16 packing), the device status
// word, bounded waits and the RoPE angle routine shared by the kernels of libqwen3attn.
#pragma once

#include <cuda.h>  // CUtensorMap (type only; the driver is reached through the runtime)
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/qwen3_attn.h"

namespace q3 {

constexpr int kD = 128;          // head_dim (the only one Qwen3 uses)
constexpr int kHalf = kD / 2;    // RoPE pairs dim i with dim i + 64

// Site codes written next to a recorded device error (which wait or check fired).
enum Site : int {
  kSiteNone = 0,
  kSitePrologueRow = 10,
  kSitePrefillQFull = 20,
  kSitePrefillKFull = 21,
  kSitePrefillVFull = 22,
  kSitePrefillKEmpty = 23,
  kSitePrefillVEmpty = 24,
  kSitePrefillSFull = 25,
  kSitePrefillPReady = 26,
  kSitePrefillOFull = 27,
  kSitePrefillDrain = 28,
  kSitePrefillQEmpty = 29,
  kSiteDecodeFull = 40,
  kSiteDecodeEmpty = 41,
  kSiteDecodeLen = 42,
  kSitePagedTable = 50,
  kSiteQkvFull = 60,
  kSiteQkvEmpty = 61,
  kSiteQkvAcc = 62,
  kSiteQkvRope = 63,
  kSiteQkvDrain = 64,
};

// Device status word: [0] = first qwen3_status recorded, [1] = its site.
__device__ int g_status[2];
// Id of the last launch in which some wait ran out: every other CTA of that launch stops
// waiting at once instead of running out its own limit.  Ids are unique per launch, so a
// stale value never affects later launches.
__device__ unsigned long long g_abort_launch;

struct WaitCfg {
  uint64_t limit_ns;   // bound on one wait
  uint64_t launch_id;  // unique per launch (host counter)
};

__device__ __forceinline__ void record_error(int code, int site) {
  if (atomicCAS(&g_status[0], 0, code) == 0) atomicExch(&g_status[1], site);
}

// ---------------------------------------------------------------------------- RoPE
// inv_i = theta^(-2i/d) split as hi + lo (two floats, computed on the host in double),
// so pos * inv_i can be formed to ~2^-48 relative with fp32 FMAs.
struct RopeTable {
  float hi[kHalf];
  float lo[kHalf];
};

// sin/cos of pos * inv_i with |angle error| <~ 5e-7 rad for |pos| < 2^24.
// Product: p = fl(pos*hi) plus its exact FMA residual and the lo term.  Reduction modulo
// 2*pi: two-term Cody-Waite with fused multiply-add (the first step is exact because
// p - n*C1 needs at most 23 significant bits).  sincosf on the reduced argument is the
// accurate libm routine, not the fast intrinsic.
__device__ __forceinline__ void rope_sincos(int pos, float hi, float lo, float& s, float& c) {
  const float fp = static_cast<float>(pos);
  const float p = __fmul_rn(fp, hi);
  const float e = fmaf(fp, hi, -p);
  const float t = fmaf(fp, lo, e);
  const float kInv2Pi = 0.159154943091895336f;
  const float kC1 = 6.28318548202514648f;     // float nearest 2*pi
  const float kC2 = -1.74845553146951657e-07f; // 2*pi - kC1
  const float n = rintf(__fmul_rn(p, kInv2Pi));
  float r = fmaf(-n, kC1, p);
  r = fmaf(-n, kC2, r);
  r = __fadd_rn(r, t);
  sincosf(r, &s, &c);
}

// Programmatic dependent launch.  A kernel launched with programmatic stream serialization
// may start while the previous kernel in the stream still runs; griddep_wait() blocks the
// calling thread until that kernel has completed and its memory writes are visible (a
// no-op when there is no such kernel).  griddep_launch_dependents() lets the next kernel
// start once every CTA of this grid has issued it or exited.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------------------- bf16
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  // cvt.rn.bf16x2.f32 d, a, b puts a in the upper half and b in the lower half.
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
__device__ __forceinline__ float bf16lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

// ---------------------------------------------------------------------------- smem / mbarrier
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_init_fence() {
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
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Non-blocking probe of an mbarrier phase (no suspension).
__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// The waiting part of mbar_wait, out of line so the common already-complete case costs
// one inline probe rather than a call.
__device__ __noinline__ bool mbar_wait_slow(uint32_t bar, uint32_t parity, uint64_t limit_ns, uint64_t launch_id,
                                            volatile int* abort, int site) {
  const uint64_t t0 = global_timer_ns();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 15u) == 0u) {
      if (abort != nullptr) {
        if (*abort != 0) return false;
        if (*reinterpret_cast<volatile unsigned long long*>(&g_abort_launch) == launch_id) {
          *abort = 1;
          return false;
        }
      }
      if (global_timer_ns() - t0 > limit_ns) {
        record_error(QWEN3_ERR_DEVICE_TIMEOUT, site);
        atomicExch(&g_abort_launch, static_cast<unsigned long long>(launch_id));
        if (abort != nullptr) *abort = 1;
        return false;
      }
    }
  }
}

// Bounded wait on an mbarrier phase.  Returns false when the wait ran out (the error is
// recorded, *abort is raised so the other roles of this CTA stop, and the launch is marked
// so the other CTAs stop too), or when this CTA or launch has already aborted.  Pass
// abort == nullptr to wait regardless (used when draining copies still in flight).
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, const WaitCfg& w, volatile int* abort,
                                          int site) {
  if (mbar_test(bar, parity)) return true;
  return mbar_wait_slow(bar, parity, w.limit_ns, w.launch_id, abort, site);
}

// Generic-proxy shared-memory writes -> visible to the async proxy (TMA, tcgen05.mma).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------------------- TMA
__device__ __forceinline__ void tma_prefetch_map(const CUtensorMap* m) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(m) : "memory");
}
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* m, uint32_t bar, int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(m), "r"(bar), "r"(c0), "r"(c1)
      : "memory");
}
__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap* m, uint32_t bar, int c0, int c1,
                                            int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(dst),
      "l"(m), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}

// Tiled bulk store smem -> global (out-of-range rows of the box are not written), tracked by
// the issuing thread's bulk-async groups.
__device__ __forceinline__ void tma_store_4d(const CUtensorMap* m, uint32_t src, int c0, int c1, int c2, int c3) {
  asm volatile("cp.async.bulk.tensor.4d.global.shared::cta.bulk_group [%0, {%2, %3, %4, %5}], [%1];" ::"l"(m),
               "r"(src), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
               : "memory");
}
__device__ __forceinline__ void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until every committed bulk store of this thread has finished reading shared memory.
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// Wait until every committed bulk store of this thread has completed.
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// ---------------------------------------------------------------------------- tcgen05
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
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Arrive once on `bar` when every tcgen05 operation this thread issued so far completes.
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}
// D[tmem] (+)= A[smem desc] * B[smem desc], bf16 inputs, fp32 accumulate.
__device__ __forceinline__ void tc_mma_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Shared-memory matrix descriptor for a 128-byte-swizzled operand (sm100 layout):
// start address, leading/stride byte offsets (all >> 4), version 1, swizzle mode 2.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) | (static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16) |
         (static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor, kind::f16: bf16 A and B, fp32 D, dense, A K-major.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((b_mn_major ? 1u : 0u) << 16) |
         (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

#define Q3_R8(i) "=r"(r[i]), "=r"(r[i + 1]), "=r"(r[i + 2]), "=r"(r[i + 3]), "=r"(r[i + 4]), "=r"(r[i + 5]), \
                 "=r"(r[i + 6]), "=r"(r[i + 7])
#define Q3_S8(i) "r"(r[i]), "r"(r[i + 1]), "r"(r[i + 2]), "r"(r[i + 3]), "r"(r[i + 4]), "r"(r[i + 5]), \
                 "r"(r[i + 6]), "r"(r[i + 7])

// 32 lanes x 32 consecutive fp32 columns: thread t of the warp gets lane (quadrant*32 + t).
// The load and its wait are one asm statement so no use of r[] can move above the wait.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n\t"
      "tcgen05.wait::ld.sync.aligned;\n"
      : Q3_R8(0), Q3_R8(8), Q3_R8(16), Q3_R8(24)
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};\n\t"
      "tcgen05.wait::st.sync.aligned;\n" ::"r"(taddr),
      Q3_S8(0), Q3_S8(8), Q3_S8(16), Q3_S8(24)
      : "memory");
}

// 32 lanes x 32 columns, no wait: the registers are not valid until tmem_wait_ld_dep(r).
__device__ __forceinline__ void tmem_ld32_nowait(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n"
      : Q3_R8(0), Q3_R8(8), Q3_R8(16), Q3_R8(24)
      : "r"(taddr)
      : "memory");
}
#define Q3_RW8(i) "+r"(r[i]), "+r"(r[i + 1]), "+r"(r[i + 2]), "+r"(r[i + 3]), "+r"(r[i + 4]), "+r"(r[i + 5]), \
                  "+r"(r[i + 6]), "+r"(r[i + 7])
// Wait for outstanding TMEM loads; naming r as read-write keeps every use of r below it.
__device__ __forceinline__ void tmem_wait_ld_dep(uint32_t (&r)[32]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;\n" : Q3_RW8(0), Q3_RW8(8), Q3_RW8(16), Q3_RW8(24) : : "memory");
}
// 32 lanes x 16 columns, with its wait.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n\t"
      "tcgen05.wait::ld.sync.aligned;\n"
      : Q3_R8(0), Q3_R8(8)
      : "r"(taddr)
      : "memory");
}

// 32 lanes x 64 consecutive fp32 columns in one load, with its wait.
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, uint32_t (&r)[64]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x64.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,"
      "%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,"
      "%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%64];\n\t"
      "tcgen05.wait::ld.sync.aligned;\n"
      : Q3_R8(0), Q3_R8(8), Q3_R8(16), Q3_R8(24), Q3_R8(32), Q3_R8(40), Q3_R8(48), Q3_R8(56)
      : "r"(taddr)
      : "memory");
}

// 32 lanes x 128 consecutive fp32 columns in one load, with its wait.
__device__ __forceinline__ void tmem_ld128(uint32_t taddr, uint32_t (&r)[128]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x128.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,"
      "%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,"
      "%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63,"
      "%64,%65,%66,%67,%68,%69,%70,%71,%72,%73,%74,%75,%76,%77,%78,%79,"
      "%80,%81,%82,%83,%84,%85,%86,%87,%88,%89,%90,%91,%92,%93,%94,%95,"
      "%96,%97,%98,%99,%100,%101,%102,%103,%104,%105,%106,%107,%108,%109,%110,%111,"
      "%112,%113,%114,%115,%116,%117,%118,%119,%120,%121,%122,%123,%124,%125,%126,%127}, [%128];\n\t"
      "tcgen05.wait::ld.sync.aligned;\n"
      : Q3_R8(0), Q3_R8(8), Q3_R8(16), Q3_R8(24), Q3_R8(32), Q3_R8(40), Q3_R8(48), Q3_R8(56), Q3_R8(64),
        Q3_R8(72), Q3_R8(80), Q3_R8(88), Q3_R8(96), Q3_R8(104), Q3_R8(112), Q3_R8(120)
      : "r"(taddr)
      : "memory");
}

// Packed fp32 pairs (sm_100 f32x2 arithmetic: one instruction for two lanes of work).
__device__ __forceinline__ uint64_t f2pack(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void f2unpack(uint64_t v, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t fadd2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t fmul2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// 32 lanes x 16 consecutive 32-bit columns, no wait: pair with tmem_wait_st().
__device__ __forceinline__ void tmem_st16_nowait(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};\n" ::"r"(taddr),
      Q3_S8(0), Q3_S8(8)
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}
__device__ __forceinline__ void st_shared_u32(uint32_t addr, uint32_t a) {
  asm volatile("st.shared.b32 [%0], %1;" ::"r"(addr), "r"(a) : "memory");
}

// Offset of the 16-byte chunk `chunk` (0..7) of row `row` inside a 128B-swizzled tile
// whose rows are 128 bytes: the chunk index is XORed with the row index modulo 8.
__device__ __forceinline__ uint32_t sw128_offset(uint32_t row, uint32_t chunk) {
  return row * 128u + ((chunk ^ (row & 7u)) << 4);
}

// AND of v over the 128 threads of named barrier `id` (bar.red: a barrier that also reduces).
__device__ __forceinline__ bool group_all(int id, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred pi, po;\n\t"
      "setp.ne.u32 pi, %1, 0;\n\t"
      "bar.red.and.pred po, %2, 128, pi;\n\t"
      "selp.u32 %0, 1, 0, po;\n\t}\n"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v)), "r"(id)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// QK-Norm + RoPE of one head vector held by a warp: lane l owns dims {2l, 2l+1} (xa) and
// {64+2l, 65+2l} (xb).  Returns the rotated, normalised pairs (fp32) for the same dims.
// g: gain; (s0,c0),(s1,c1): sin/cos of the angles of frequencies 2l and 2l+1.
__device__ __forceinline__ void norm_rope_pairs(float2 xa, float2 xb, float2 ga, float2 gb, float s0, float c0,
                                                float s1, float c1, float eps, float2& ya, float2& yb) {
  float ss = xa.x * xa.x + xa.y * xa.y + xb.x * xb.x + xb.y * xb.y;
  ss = warp_sum(ss);
  const float r = rsqrtf(fmaf(ss, 1.0f / kD, eps));
  const float a0 = ga.x * (xa.x * r), a1 = ga.y * (xa.y * r);
  const float b0 = gb.x * (xb.x * r), b1 = gb.y * (xb.y * r);
  ya.x = a0 * c0 - b0 * s0;
  yb.x = b0 * c0 + a0 * s0;
  ya.y = a1 * c1 - b1 * s1;
  yb.y = b1 * c1 + a1 * s1;
}

}  // namespace q3
