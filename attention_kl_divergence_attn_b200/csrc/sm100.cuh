// sm100.cuh — thin inline-PTX wrappers for the Blackwell (sm_100a) features the
// attention-KL kernels use: mbarriers, TMA tile loads, tcgen05 tensor-memory
// allocation, MMA, commit, loads/stores and fences, and the shared-memory /
// instruction descriptors of tcgen05.mma.  Every wait is bounded: it gives up
// after a wall-clock budget, records a status code and lets the caller unwind.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

namespace skl {

// ---------------------------------------------------------------- status word
// Bit layout of the device status word that lives in the caller's workspace.
enum : uint32_t {
    kStatusTimeout = 1u << 0,   // some bounded wait gave up
    kStatusBadLength = 1u << 1, // a per-batch key length outside [0, N_K] (clamped)
    kStatusBounds = 1u << 2,    // bounds-checked build: an access outside its tensor (skipped)
    kStatusWhoShift = 8,        // bits 8..15: which wait (role-specific id)
    kStatusSiteShift = 16,      // bits 16..23: which checked access (bounds-checked build)
};

// ---------------------------------------------------------------- bounds-checked build
// Built with STREAMKL_CHECK_BOUNDS (libstreamkl_checked.so), every TMA
// coordinate and every global index that the kernels compute is checked
// against its tensor before the access; a violation skips the access and ORs
// kStatusBounds and the site's id into the status word (nothing traps, and a
// skipped copy ends in a bounded wait that gives up).  Otherwise the checks
// compile to nothing.
#ifdef STREAMKL_CHECK_BOUNDS
constexpr bool kCheckBounds = true;
#else
constexpr bool kCheckBounds = false;
#endif

// Site ids of the checked accesses.
enum : uint32_t {
    kSiteTma = 1, kSiteRowOut = 2, kSiteDrain = 3, kSiteResident = 4, kSiteConst = 5, kSiteZero = 6,
};

// true when `ok` (always in an unchecked build); otherwise records the site.
__device__ __forceinline__ bool bound_ok(bool ok, uint32_t *word, uint32_t site) {
    if constexpr (kCheckBounds) {
        if (!ok) {
            if (word) atomicOr(word, kStatusBounds | (site << kStatusSiteShift));
            return false;
        }
    }
    return true;
}

// Extent of the tensor behind one TMA map: n0 columns (the head dimension),
// n1 rows, n2 heads.
struct MapDims {
    int n0, n1, n2;
};

struct DevStatus {
    uint32_t *word;             // device status word (workspace)
    unsigned long long budget_ns;
};

// ---------------------------------------------------------------- problem geometry
// Grouped key heads: query head bh = b * H + h reads key head
// b * Hk + h / (H / Hk) of a key tensor with Hk heads per batch element.
__device__ __forceinline__ int key_head(int bh, int H, int Hk) { return (bh / H) * Hk + (bh % H) / (H / Hk); }

// Keys of batch element b that are not padding: kv_len[b] clamped to
// [0, N_K] (all N_K without lengths).  With `report`, a length outside that
// range sets kStatusBadLength in the status word.
__device__ __forceinline__ int key_count(const int *kv_len, int b, int N_K, uint32_t *word, bool report) {
    if (!kv_len) return N_K;
    const int len = __ldg(kv_len + b);
    if (report && (len < 0 || len > N_K) && word) atomicOr(word, (uint32_t)kStatusBadLength);
    return len < 0 ? 0 : (len > N_K ? N_K : len);
}

// Item r of a persistent CTA: items (head, row tile) are numbered heaviest
// first and dealt out in rounds of gridDim.x, alternately left to right and
// right to left, so that every CTA gets a similar share of heavy and light
// items; -1 once this CTA has none left.
__device__ __forceinline__ int persistent_item(int r, int n_items) {
    const long long base = (long long)r * gridDim.x;
    const long long j = base + ((r & 1) ? (int)(gridDim.x - 1 - blockIdx.x) : (int)blockIdx.x);
    return j < n_items ? (int)j : -1;
}

__device__ __forceinline__ unsigned long long globaltimer() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ bool elect_one() {
    uint32_t pred = 0;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "elect.sync _|p, 0xffffffff;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(pred));
    return pred != 0;
}

// ---------------------------------------------------------------- global loads
// A read-only global load issued exactly here (volatile: the compiler may not
// sink it towards its first use, which would defeat a software prefetch).
__device__ __forceinline__ float ld_now(const float *p) {
    float v;
    asm volatile("ld.global.nc.f32 %0, [%1];" : "=f"(v) : "l"(p));
    return v;
}

// 32-byte global store (one whole sector; `p` must be 32-byte aligned).
__device__ __forceinline__ void st_global_v8(float *p, float a, float b, float c, float d, float e, float f, float g,
                                             float h) {
    asm volatile("st.global.v8.f32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "f"(a), "f"(b), "f"(c), "f"(d),
                 "f"(e), "f"(f), "f"(g), "f"(h)
                 : "memory");
}

// Asks L2 to fetch `bytes` (a multiple of 16) of global memory starting at the
// 16-byte aligned `p`, without waiting (a hint: nothing is written anywhere).
__device__ __forceinline__ void prefetch_l2(const void *p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait for the phase with the given parity to complete.  Returns false
// (after recording the timeout in the status word and raising the CTA's abort
// flag) when the budget runs out or another role of the CTA already aborted.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, const DevStatus &st,
                                          volatile int *abort_flag, uint32_t who) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = globaltimer();
    for (uint32_t spin = 1;; ++spin) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((spin & 63u) == 0) {
            if (*abort_flag) return false;
            if (globaltimer() - t0 > st.budget_ns) {
                *abort_flag = 1;
                if (st.word) atomicOr(st.word, kStatusTimeout | (who << kStatusWhoShift));
                return false;
            }
        }
    }
}

// ---------------------------------------------------------------- fences
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Named barrier `id` over `n` threads (a multiple of 32) that also returns,
// to every one of them, whether any of them passed `pred` true: a decision
// all participants take alike.
// Named CTA barriers (bar.sync / bar.arrive, aligned: every lane of a warp
// executes them; n counts threads, a multiple of 32).
__device__ __forceinline__ void named_sync(int id, int n) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}
__device__ __forceinline__ void named_arrive(int id, int n) {
    asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(n) : "memory");
}

__device__ __forceinline__ bool bar_sync_or(int id, int n, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)pred), "r"(id), "r"(n)
        : "memory");
    return r != 0;
}

// ---------------------------------------------------------------- TMA
// 3-D tiled load (coordinates innermost first) into shared memory, completing
// transaction bytes on `bar`.  The innermost coordinate is always a multiple
// of 64 elements here, so its byte offset is 16-byte aligned.  `dims` is the
// map's tensor and `word` the status word, used by the bounds-checked build:
// the innermost coordinate a multiple of 64 inside the row, the box's first
// row inside the tensor (later rows past its end are the zero-filled tail),
// the head in range.
__device__ __forceinline__ void tma_load_3d(void *dst, const CUtensorMap *map, uint64_t *bar, int c0,
                                            int c1, int c2, MapDims dims, uint32_t *word) {
    if (!bound_ok(c0 >= 0 && (c0 & 63) == 0 && c0 + 64 <= dims.n0 && c1 >= 0 && c1 < dims.n1 && c2 >= 0 &&
                      c2 < dims.n2,
                  word, kSiteTma))
        return;
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap *map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ---------------------------------------------------------------- TMEM
// Allocation is warp-wide; the base column address is written to *dst (smem).
__device__ __forceinline__ void tmem_alloc(uint32_t *dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)),
                 "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T  (kind::f16, bf16 inputs, fp32 accumulate).
__device__ __forceinline__ void mma_bf16_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]^T: A is read from tensor memory (M lanes x K
// bf16, two elements per 32-bit column, K-major), B from shared memory.
__device__ __forceinline__ void mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive (once) on `bar` when every MMA issued so far by this thread is done.
__device__ __forceinline__ void mma_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

// Before a CTA frees its tensor memory, every MMA that this thread issued must
// have completed.  On the normal path they have (their results were read);
// on a path that gave up early some may still be running.  The thread
// commits to `bar` (an mbarrier for this one use, one arrival) and waits for
// it with a short bounded wait of its own.
__device__ __forceinline__ void mma_quiesce(uint64_t *bar, const DevStatus &st, uint32_t who) {
    mma_commit(bar);
    DevStatus quick = st;
    quick.budget_ns = 50000000ull;
    volatile int never = 0;
    mbar_wait(bar, 0, quick, &never, who);
}

// 32 lanes x 32 consecutive fp32 columns: thread t of the warp gets lane
// (warp's lane quarter base + t), columns [col, col+32).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
          "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
          "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
          "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
#pragma unroll
    for (int k = 0; k < 32; ++k) v[k] = __uint_as_float(r[k]);
}

// 32 lanes x 16 consecutive fp32 columns (see tmem_ld32).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
#pragma unroll
    for (int k = 0; k < 16; ++k) v[k] = __uint_as_float(r[k]);
}

__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// 32 lanes x 8 consecutive fp32 columns (see tmem_ld32).
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float (&v)[8]) {
    uint32_t r[8];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
#pragma unroll
    for (int k = 0; k < 8; ++k) v[k] = __uint_as_float(r[k]);
}

// tcgen05.wait::ld that also names the registers the outstanding loads fill,
// so that the compiler cannot schedule a use of them ahead of the wait (a
// plain wait orders memory only).  Used when a load is issued one step ahead
// of the code that consumes it.
__device__ __forceinline__ void tmem_ld_wait_bind(float (&a)[8], float (&b)[8]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+f"(a[0]), "+f"(a[1]), "+f"(a[2]), "+f"(a[3]), "+f"(a[4]), "+f"(a[5]), "+f"(a[6]), "+f"(a[7]),
                   "+f"(b[0]), "+f"(b[1]), "+f"(b[2]), "+f"(b[3]), "+f"(b[4]), "+f"(b[5]), "+f"(b[6]), "+f"(b[7])
                 :
                 : "memory");
}
__device__ __forceinline__ void tmem_ld_wait_bind(float (&a)[16], float (&b)[16]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+f"(a[0]), "+f"(a[1]), "+f"(a[2]), "+f"(a[3]), "+f"(a[4]), "+f"(a[5]), "+f"(a[6]), "+f"(a[7]),
                   "+f"(a[8]), "+f"(a[9]), "+f"(a[10]), "+f"(a[11]), "+f"(a[12]), "+f"(a[13]), "+f"(a[14]),
                   "+f"(a[15]), "+f"(b[0]), "+f"(b[1]), "+f"(b[2]), "+f"(b[3]), "+f"(b[4]), "+f"(b[5]), "+f"(b[6]),
                   "+f"(b[7]), "+f"(b[8]), "+f"(b[9]), "+f"(b[10]), "+f"(b[11]), "+f"(b[12]), "+f"(b[13]),
                   "+f"(b[14]), "+f"(b[15])
                 :
                 : "memory");
}
// Width-generic wrappers (8 or 16 columns).
template <int W>
__device__ __forceinline__ void tmem_ld(uint32_t taddr, float (&v)[W]) {
    static_assert(W == 8 || W == 16, "8 or 16 columns");
    if constexpr (W == 8) tmem_ld8(taddr, v); else tmem_ld16(taddr, v);
}

// 32 lanes x 16 consecutive 32-bit columns: thread t of the warp writes lane
// (warp's lane quarter base + t), columns [col, col+16).
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
        "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
        : "memory");
}

// 32 lanes x 8 consecutive 32-bit columns (see tmem_st16).
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t *v) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), "r"(v[0]),
                 "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
                 : "memory");
}

// 32 lanes x 4 consecutive 32-bit columns (see tmem_st16).
__device__ __forceinline__ void tmem_st4(uint32_t taddr, const uint32_t *v) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1,%2,%3,%4};" ::"r"(taddr), "r"(v[0]), "r"(v[1]),
                 "r"(v[2]), "r"(v[3])
                 : "memory");
}

__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// ---------------------------------------------------------------- descriptors
// Shared-memory matrix descriptor of tcgen05.mma for a 128-byte-swizzled
// operand.  `lbo`/`sbo` are byte offsets: for a K-major operand the stride
// between 8-row groups is sbo (lbo unused); for an MN-major operand lbo is the
// stride between 64-element MN blocks and sbo the stride between 8-row K groups.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t smem_addr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= (uint64_t)((smem_addr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;                 // descriptor version (sm_100)
    d |= (uint64_t)2 << 61;                 // 128-byte swizzle
    return d;
}

// Shared-memory matrix descriptor of tcgen05.mma for an unswizzled K-major
// operand of 16-element rows: 8-row x 16-byte core matrices, `lbo` bytes between
// the two core matrices of a row block (K elements 0-7 and 8-15), `sbo` bytes
// between 8-row blocks.
__device__ __forceinline__ uint64_t plain_desc(uint32_t smem_addr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= (uint64_t)((smem_addr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;                 // descriptor version (sm_100), no swizzle
    return d;
}

// A descriptor advanced by `bytes` (a multiple of 16): the start address lives in
// the low 14 bits in 16-byte units, and shared-memory addresses stay below 256 KB,
// so the add never carries into the other fields.
__device__ __forceinline__ uint64_t desc_add(uint64_t desc, uint32_t bytes) { return desc + (uint64_t)(bytes >> 4); }

// Instruction descriptor: bf16 x bf16 -> fp32, dense, M x N, operand majors
// (0 = K-major, 1 = MN-major).
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, int a_mn, int b_mn) {
    return (1u << 4)                        // D format fp32
           | (1u << 7)                      // A format bf16
           | (1u << 10)                     // B format bf16
           | ((uint32_t)a_mn << 15) | ((uint32_t)b_mn << 16)
           | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// ---------------------------------------------------------------- math
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float lg2(float x) {
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// One 16-byte shared-memory load issued exactly here (`p` 16-byte aligned).
__device__ __forceinline__ float4 ld_shared_v4(const float *p) {
    float4 v;
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(smem_u32(p)));
    return v;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// ---------------------------------------------------------------- packed fp32 pairs
// Two fp32 values in one 64-bit register pair (low half = first value); the
// .f32x2 instructions process both with one issue slot.
__device__ __forceinline__ uint64_t f2pack(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ float2 f2unpack(uint64_t v) {
    float2 r;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(v));
    return r;
}
__device__ __forceinline__ uint64_t f2add(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("add.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t f2sub(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("sub.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t f2mul(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("mul.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t f2fma(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}
__device__ __forceinline__ uint64_t f2splat(float v) { return f2pack(v, v); }
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}
// 2^x of both halves on the ex2 unit.
__device__ __forceinline__ uint64_t ex2_pair(uint64_t x) {
    const float2 v = f2unpack(x);
    return f2pack(ex2(v.x), ex2(v.y));
}

// Copies this thread's row of a bf16 [rows][D] tensor into W columns of its
// TMEM lane (two elements per 32-bit column, lower element in the low half:
// the layout of an A operand that tcgen05.mma reads from tensor memory).
// `src` points at the first of the 2W elements, or is null for a row past the
// end of the tensor, which gets zeros.
template <int W>
__device__ __forceinline__ void row_to_tmem(uint32_t taddr, const __nv_bfloat16 *src) {
    static_assert(W == 8 || W == 16, "8 or 16 columns");
    uint32_t v[W];
    const uint4 *s4 = reinterpret_cast<const uint4 *>(src);
#pragma unroll
    for (int k = 0; k < W / 4; ++k) {
        const uint4 x = src ? __ldg(s4 + k) : make_uint4(0u, 0u, 0u, 0u);
        v[4 * k] = x.x; v[4 * k + 1] = x.y; v[4 * k + 2] = x.z; v[4 * k + 3] = x.w;
    }
    if constexpr (W == 16) tmem_st16(taddr, v); else tmem_st8(taddr, v);
}

// Every one of four warpgroups copies a quarter of the columns of one resident
// 128-row operand (rows row0 .. row0+127 of head bh of a [nheads, N, D]
// tensor) into tensor memory at column `col`; warp `sub` of a warpgroup must
// be an SM sub-partition's warp (warp index mod 4), which may touch only lanes
// 32*sub .. 32*sub+31.
template <int D>
__device__ __forceinline__ void resident_to_tmem(uint32_t tmem, uint32_t col, const void *base, int bh, int N, int row0,
                                                 int wg, int sub, int lane, int nheads, uint32_t *word) {
    constexpr int W = D / 2 / 4;
    const int r = row0 + sub * 32 + lane;
    const bool in = r < N && bound_ok(bh >= 0 && bh < nheads && r >= 0 && wg >= 0 && wg < 4, word, kSiteResident);
    const __nv_bfloat16 *src =
        in ? static_cast<const __nv_bfloat16 *>(base) + ((size_t)bh * N + r) * D + wg * 2 * W : nullptr;
    row_to_tmem<W>(tmem + ((uint32_t)(sub * 32) << 16) + col + wg * W, src);
}

// Byte offset of element (row, col) in a [rows][64] bf16 tile stored with the
// 128-byte swizzle that TMA (CU_TENSOR_MAP_SWIZZLE_128B) and tcgen05 share:
// the 16-byte chunk index is XORed with (row mod 8).  Tile base 1024-aligned.
__device__ __forceinline__ uint32_t sw128_offset(uint32_t row, uint32_t col) {
    return row * 128u + ((((col >> 3) ^ (row & 7u)) & 7u) << 4) + ((col & 7u) << 1);
}

// Copies warpgroup wg's quarter of one row of a TMA-loaded 128-row bf16 tile
// (D/64 boxes of [128 rows][64], 128-byte swizzle) into tensor memory at
// `taddr` (this warp's lane base plus the operand's column): columns
// wg*W .. wg*W+W-1 of the packed row, W = D/8, two elements per column with
// the lower element in the low half (the A-operand layout of tcgen05.mma).
template <int D>
__device__ __forceinline__ void tile_rows_to_tmem(uint32_t taddr, const uint8_t *tile, int wg, int row) {
    constexpr int W = D / 2 / 4;
    uint32_t v[W];
#pragma unroll
    for (int k = 0; k < W / 4; ++k) {
        const int e = wg * 2 * W + k * 8;     // first of the chunk's 8 elements
        const uint4 x = *reinterpret_cast<const uint4 *>(tile + (e / 64) * (128 * 128) + sw128_offset(row, e % 64));
        v[4 * k] = x.x; v[4 * k + 1] = x.y; v[4 * k + 2] = x.z; v[4 * k + 3] = x.w;
    }
    if constexpr (W == 16) tmem_st16(taddr + wg * W, v); else tmem_st8(taddr + wg * W, v);
}

}  // namespace skl
