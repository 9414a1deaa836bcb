// fwd.cuh — one-pass forward of the attention-distillation KL divergence.
//
// Source: "StreamKL: Fast and Memory-Efficient KL Divergence for Boosting
// Attention Distillation", abstract — a single forward kernel that streams
// query-key tiles through on-chip memory with an online formulation of the
// coupled two-distribution KL reduction, so neither softmax is materialised.
//
// One CTA owns 128 query rows of one (batch, head).  Roles (2 + 4*NWG warps):
//   warp 0      TMA producer: K_t, K_s tiles of 64 keys into an NSTAGE-deep
//               shared-memory ring.
//   warp 1      MMA issuer (one elected thread) and TMEM owner: per key tile
//               S_t = Q_t K_t^T and S_s = Q_s K_s^T as tcgen05.mma (bf16 in,
//               fp32 accumulate) into one of three TMEM buffers (3 x 128 cols).
//               Q_t and Q_s sit in the last 128 TMEM columns (packed bf16) and
//               are the MMAs' A operand, so the tensor core reads only the key
//               tile from shared memory (with both operands from shared memory
//               an N = 64 MMA is bound by shared-memory bandwidth).
//   warps 2..   4 softmax warpgroups: 2 parities in ping-pong x 2 column halves.
//               They first copy the CTA's query rows into tensor memory (each
//               warp a quarter of the columns of its 32 rows).  Warpgroup (p, h)
//               then owns key tiles p, p+2, ... and, of each, the 32 key columns
//               of half h; while a parity works on one buffer the MMA warp
//               fills the next free one.
//               Four warps per SM sub-partition keep the ex2 unit fed.  Thread = query row
//               = TMEM lane; it reads its row of both logit tiles in 32-column
//               chunks (tcgen05.ld 32x32b) and updates its own per-row online
//               state (M_t, l_t, A, M_s, l_s); row reductions are thread-local
//               because the 32x32b layout gives each thread one whole row.
//               The warpgroups' states are merged at the end (the state is
//               associative: rescale both to the larger maximum).
// State (log2 units, y = scale * log2(e) * q.k):
//   M_t, M_s  running maxima of y_t, y_s
//   l_t = sum 2^(y_t - M_t),  l_s = sum 2^(y_s - M_s)
//   A   = sum 2^(y_t - M_t) (y_t - y_s)
// and at the end LSE = ln2 (M + log2 l), KL = ln2 (A / l_t) - LSE_t + LSE_s.
// Fully masked key tiles (above the causal diagonal) are never loaded.
#pragma once

#include "sm100.cuh"

namespace skl {

struct FwdParams {
    int BH, N_Q, N_K, causal, n_qt;
    int H, Hkt, Hks;       // query heads per batch element, key heads of K_t and K_s
    const int *kv_len;     // per-batch key lengths (padding), or null
    int splits;            // key ranges per query tile (1 = the whole row in one CTA)
    float ct, cs;          // scale_t * log2(e), scale_s * log2(e)
    float *kl, *lse_t, *lse_s;
    float *part;           // splits > 1: partial states, field f of split s, row r at [(f*splits + s)*rows + r]
    DevStatus st;
};

// Online state of one row over a set of keys (log2 units, see above).
struct RowState {
    float Mt, Ms, lt, ls, A;
};

// Folds state b into a: both rescaled to the larger maxima (teacher maximum
// for l_t and A, student maximum for l_s).  Associative and exact up to
// rounding; a state with no visible key (M = -inf, sums 0) is the identity.
__device__ __forceinline__ void merge_state(RowState &a, const RowState &b) {
    const float nMt = fmaxf(a.Mt, b.Mt), nMs = fmaxf(a.Ms, b.Ms);
    if (nMt == -INFINITY) return;
    const float a1 = ex2(a.Mt - nMt), a2 = ex2(b.Mt - nMt);
    const float b1 = ex2(a.Ms - nMs), b2 = ex2(b.Ms - nMs);
    a.lt = a.lt * a1 + b.lt * a2;
    a.A = a.A * a1 + b.A * a2;
    a.ls = a.ls * b1 + b.ls * b2;
    a.Mt = nMt;
    a.Ms = nMs;
}

// Row outputs from a complete state: LSE = ln2 (M + log2 l) for each
// distribution and KL = ln2 (A / l_t) - LSE_t + LSE_s.  A row that saw no key
// (all keys padding) has the empty sums: KL = 0, LSE = -inf.
__device__ __forceinline__ void finish_row(const RowState &x, float *kl, float *lse_t, float *lse_s) {
    const float LN2 = 0.69314718055994530942f;
    if (x.lt == 0.f) {
        *kl = 0.f;
        *lse_t = -INFINITY;
        *lse_s = -INFINITY;
        return;
    }
    const float lse_t2 = x.Mt + lg2(x.lt), lse_s2 = x.Ms + lg2(x.ls);
    *lse_t = lse_t2 * LN2;
    *lse_s = lse_s2 * LN2;
    *kl = LN2 * (x.A / x.lt - lse_t2 + lse_s2);
}

// Deepest key-tile ring the forward uses.
constexpr int kFwdMaxStages = 4;

template <int DT, int DS, int NWG>
struct FwdCfg {
    static constexpr int BM = 128, BN = 64;                  // query rows per CTA, keys per tile
    static constexpr int BLK = 128 * 128;                    // one [128 rows][64] bf16 box (Q)
    static constexpr int KBLK = BN * 128;                    // one [64 rows][64] bf16 box (K)
    static constexpr int NBUF = 3;                           // TMEM logit buffers (S_t, S_s: 64 cols each)
    // the query tile's rows, packed bf16, after the logit buffers: the logit
    // MMAs take A from tensor memory and read only the key tile from shared
    // memory
    static constexpr uint32_t TMEM_QT = NBUF * 128, TMEM_QS = TMEM_QT + DT / 2;
    static constexpr int QT_BYTES = BM * DT * 2, QS_BYTES = BM * DS * 2;
    static constexpr int KT_BYTES = BN * DT * 2, KS_BYTES = BN * DS * 2;
    static constexpr int Q_BYTES = QT_BYTES + QS_BYTES;
    static constexpr int STAGE_BYTES = KT_BYTES + KS_BYTES;
    static constexpr int NS_RAW = (200 * 1024 - Q_BYTES) / STAGE_BYTES;
    static constexpr int NSTAGE = NS_RAW < 2 ? 2 : (NS_RAW > kFwdMaxStages ? kFwdMaxStages : NS_RAW);
    static constexpr int SMEM = Q_BYTES + NSTAGE * STAGE_BYTES + 1024;
    static constexpr int NH = NWG / 2;                       // column halves per parity
    static constexpr int CW = BN / NH;                       // key columns per warpgroup and tile
    static constexpr int THREADS = 64 + 128 * NWG;           // TMA warp, MMA warp, NWG softmax warpgroups
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr uint32_t IDESC = idesc_bf16(BM, BN, 0, 0);
    static_assert(NWG == 4, "2 parities x 2 column halves; four warpgroups copy the query rows");
    static_assert(TMEM_QS + DS / 2 <= TMEM_COLS, "logit buffers and query rows fit tensor memory");
};

// Number of key tiles a 128-row query tile starting at q0 must visit: keys
// below nk (the keys that are not padding) and, under the causal mask, at or
// below the tile's last row + off (off = N_K - N_Q).
__device__ __forceinline__ int fwd_key_tiles(int q0, int N_Q, int nk, int off, int causal, int BN) {
    int kend = nk;
    if (causal) {
        int last_row = min(q0 + 127, N_Q - 1);
        kend = min(nk, last_row + off + 1);
    }
    return (kend + BN - 1) / BN;
}

// Online update with one 32-column chunk of raw logits (u = q.k, unscaled),
// scalar form used for chunks that contain masked (hidden or padding) keys,
// which are passed in as -inf.
__device__ __forceinline__ void online_chunk_masked(float (&ut)[32], float (&us)[32], float ct, float cs, float &Mt,
                                                    float &Ms, float &lt, float &ls, float &A) {
    float m0 = fmaxf(ut[0], ut[1]), m1 = fmaxf(ut[2], ut[3]);
    float n0 = fmaxf(us[0], us[1]), n1 = fmaxf(us[2], us[3]);
#pragma unroll
    for (int k = 4; k < 32; k += 4) {
        m0 = fmaxf(m0, fmaxf(ut[k], ut[k + 1]));
        m1 = fmaxf(m1, fmaxf(ut[k + 2], ut[k + 3]));
        n0 = fmaxf(n0, fmaxf(us[k], us[k + 1]));
        n1 = fmaxf(n1, fmaxf(us[k + 2], us[k + 3]));
    }
    const float Mt_new = fmaxf(Mt, fmaxf(m0, m1) * ct);
    const float Ms_new = fmaxf(Ms, fmaxf(n0, n1) * cs);
    if (Mt_new == -INFINITY) return;      // nothing visible so far
    const float at = ex2(Mt - Mt_new), as = ex2(Ms - Ms_new);
    float st[4] = {0.f, 0.f, 0.f, 0.f}, ss[4] = {0.f, 0.f, 0.f, 0.f}, sa[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int k = 0; k < 32; ++k) {
        const float xt = fmaf(ut[k], ct, -Mt_new);
        const float xs = fmaf(us[k], cs, -Ms_new);
        const float et = ex2(xt), es = ex2(xs);
        st[k & 3] += et;
        ss[k & 3] += es;
        const float dx = (ut[k] == -INFINITY) ? 0.f : xt - xs;
        sa[k & 3] = fmaf(et, dx, sa[k & 3]);
    }
    const float sum_t = (st[0] + st[1]) + (st[2] + st[3]);
    const float sum_s = (ss[0] + ss[1]) + (ss[2] + ss[3]);
    const float sum_a = (sa[0] + sa[1]) + (sa[2] + sa[3]);
    lt = fmaf(lt, at, sum_t);
    ls = fmaf(ls, as, sum_s);
    A = fmaf(A, at, fmaf(Mt_new - Ms_new, sum_t, sum_a));
    Mt = Mt_new;
    Ms = Ms_new;
}

// The same update for a fully visible chunk, on packed fp32 pairs: the
// element-wise work issues one instruction per two keys and the chunk maxima
// use three-input max.  (Moving part of the exponentials to the FMA pipe with a
// polynomial was measured slower here: the loop is bound by ex2 and issue
// slots together, so the extra instructions cost more than the ex2 time saved.)
__device__ __forceinline__ void online_chunk(float (&ut)[32], float (&us)[32], float ct, float cs, float &Mt,
                                             float &Ms, float &lt, float &ls, float &A) {
    float m0 = fmax3(ut[0], ut[1], ut[2]), m1 = fmax3(ut[3], ut[4], ut[5]);
    float n0 = fmax3(us[0], us[1], us[2]), n1 = fmax3(us[3], us[4], us[5]);
#pragma unroll
    for (int k = 6; k < 30; k += 4) {
        m0 = fmax3(m0, ut[k], ut[k + 1]);
        m1 = fmax3(m1, ut[k + 2], ut[k + 3]);
        n0 = fmax3(n0, us[k], us[k + 1]);
        n1 = fmax3(n1, us[k + 2], us[k + 3]);
    }
    const float Mt_new = fmaxf(Mt, fmax3(m0, m1, fmaxf(ut[30], ut[31])) * ct);
    const float Ms_new = fmaxf(Ms, fmax3(n0, n1, fmaxf(us[30], us[31])) * cs);
    const float at = ex2(Mt - Mt_new), as = ex2(Ms - Ms_new);
    const uint64_t ct2 = f2splat(ct), cs2 = f2splat(cs);
    const uint64_t nMt = f2splat(-Mt_new), nMs = f2splat(-Ms_new);
    uint64_t st[2] = {0ull, 0ull}, ss[2] = {0ull, 0ull}, sa[2] = {0ull, 0ull};
#pragma unroll
    for (int k = 0; k < 32; k += 2) {
        const int j = (k >> 1) & 1;
        const uint64_t xt = f2fma(f2pack(ut[k], ut[k + 1]), ct2, nMt);
        const uint64_t xs = f2fma(f2pack(us[k], us[k + 1]), cs2, nMs);
        const uint64_t et = ex2_pair(xt);
        const uint64_t es = ex2_pair(xs);
        st[j] = f2add(st[j], et);
        ss[j] = f2add(ss[j], es);
        sa[j] = f2fma(et, f2sub(xt, xs), sa[j]);
    }
    const float2 t2 = f2unpack(f2add(st[0], st[1])), s2 = f2unpack(f2add(ss[0], ss[1]));
    const float2 a2 = f2unpack(f2add(sa[0], sa[1]));
    lt = fmaf(lt, at, t2.x + t2.y);
    ls = fmaf(ls, as, s2.x + s2.y);
    A = fmaf(A, at, fmaf(Mt_new - Ms_new, t2.x + t2.y, a2.x + a2.y));
    Mt = Mt_new;
    Ms = Ms_new;
}


// Fully visible chunk with a lagging maximum: when every row of the warp has
// its chunk maxima at most 8 (log2 units) above its running maxima M_t, M_s,
// the exponentials are taken against the running maxima unchanged (terms up
// to 2^8, exact in fp32), which skips the two rescale exponentials and the
// wait for the updated maxima; otherwise the chunk goes through online_chunk
// with the exact new maxima.
__device__ __forceinline__ void online_chunk_lag(float (&ut)[32], float (&us)[32], float ct, float cs, float &Mt,
                                                 float &Ms, float &lt, float &ls, float &A) {
    float m0 = fmax3(ut[0], ut[1], ut[2]), m1 = fmax3(ut[3], ut[4], ut[5]);
    float n0 = fmax3(us[0], us[1], us[2]), n1 = fmax3(us[3], us[4], us[5]);
#pragma unroll
    for (int k = 6; k < 30; k += 4) {
        m0 = fmax3(m0, ut[k], ut[k + 1]);
        m1 = fmax3(m1, ut[k + 2], ut[k + 3]);
        n0 = fmax3(n0, us[k], us[k + 1]);
        n1 = fmax3(n1, us[k + 2], us[k + 3]);
    }
    const float cmt = fmax3(m0, m1, fmaxf(ut[30], ut[31])) * ct;
    const float cms = fmax3(n0, n1, fmaxf(us[30], us[31])) * cs;
    const bool fits = (cmt <= Mt + 8.f) && (cms <= Ms + 8.f);
    if (__all_sync(0xffffffffu, fits)) {
        const uint64_t ct2 = f2splat(ct), cs2 = f2splat(cs);
        const uint64_t nMt = f2splat(-Mt), nMs = f2splat(-Ms);
        uint64_t st[2] = {0ull, 0ull}, ss[2] = {0ull, 0ull}, sa[2] = {0ull, 0ull};
#pragma unroll
        for (int k = 0; k < 32; k += 2) {
            const int j = (k >> 1) & 1;
            const uint64_t xt = f2fma(f2pack(ut[k], ut[k + 1]), ct2, nMt);
            const uint64_t xs = f2fma(f2pack(us[k], us[k + 1]), cs2, nMs);
            const uint64_t et = ex2_pair(xt);
            const uint64_t es = ex2_pair(xs);
            st[j] = f2add(st[j], et);
            ss[j] = f2add(ss[j], es);
            sa[j] = f2fma(et, f2sub(xt, xs), sa[j]);
        }
        const float2 t2 = f2unpack(f2add(st[0], st[1])), s2 = f2unpack(f2add(ss[0], ss[1]));
        const float2 a2 = f2unpack(f2add(sa[0], sa[1]));
        lt += t2.x + t2.y;
        ls += s2.x + s2.y;
        A += fmaf(Mt - Ms, t2.x + t2.y, a2.x + a2.y);
    } else {
        online_chunk(ut, us, ct, cs, Mt, Ms, lt, ls, A);
    }
}

template <int DT, int DS, int NWG>
__global__ void __launch_bounds__(FwdCfg<DT, DS, NWG>::THREADS, 1)
    streamkl_fwd_kernel(const __grid_constant__ CUtensorMap mQt, const __grid_constant__ CUtensorMap mKt,
                        const __grid_constant__ CUtensorMap mQs, const __grid_constant__ CUtensorMap mKs,
                        const FwdParams p) {
    using C = FwdCfg<DT, DS, NWG>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sQt = smem;                  // landing area of the query rows
    uint8_t *sQs = sQt + C::QT_BYTES;
    uint8_t *sK = sQs + C::QS_BYTES;      // stage s: K_t then K_s

    __shared__ uint64_t bar_q, bar_qtm, bar_kfull[C::NSTAGE], bar_kempty[C::NSTAGE], bar_sfull[C::NBUF], bar_sempty[C::NBUF];
    __shared__ uint64_t bar_quiet;                 // the MMA thread's issued MMAs have completed
    __shared__ uint32_t tmem_base_sh;
    __shared__ int abort_flag;
    __shared__ float merge[NWG > 1 ? NWG - 1 : 1][5][128];   // per-row states of warpgroups 1..NWG-1

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // tensors behind the four maps (bounds-checked build)
    const MapDims mdQt{DT, p.N_Q, p.BH}, mdQs{DS, p.N_Q, p.BH};
    const MapDims mdKt{DT, p.N_K, p.BH / p.H * p.Hkt}, mdKs{DS, p.N_K, p.BH / p.H * p.Hks};
    // heaviest (latest) causal query tiles first; with key splits, the splits
    // of one query tile are adjacent in launch order
    const int lin = (int)(blockIdx.x / p.BH);
    const int split = lin % p.splits;
    const int qt_idx = p.n_qt - 1 - lin / p.splits;
    const int bh = (int)(blockIdx.x % p.BH);
    const int q0 = qt_idx * C::BM;
    const int off = p.N_K - p.N_Q;
    // keys of this head: its key heads (grouped key heads) and its batch
    // element's keys that are not padding
    const int bkt = key_head(bh, p.H, p.Hkt), bks = key_head(bh, p.H, p.Hks);
    const int nk = key_count(p.kv_len, bh / p.H, p.N_K, p.st.word, threadIdx.x == 0 && split == 0);
    const int n_all = fwd_key_tiles(q0, p.N_Q, nk, off, p.causal, C::BN);
    // this CTA's key tiles [kt_lo, kt_lo + n_kt); loops below count from 0
    const int kt_lo = (int)((long long)n_all * split / p.splits);
    const int n_kt = (int)((long long)n_all * (split + 1) / p.splits) - kt_lo;

    if (threadIdx.x == 0) {
        mbar_init(&bar_q, 1);
        mbar_init(&bar_qtm, 4 * NWG);    // every softmax warp, once its query rows are in tensor memory
        for (int s = 0; s < C::NSTAGE; ++s) {
            mbar_init(&bar_kfull[s], 1);
            mbar_init(&bar_kempty[s], 1);
        }
        for (int b = 0; b < C::NBUF; ++b) {
            mbar_init(&bar_sfull[b], 1);
            mbar_init(&bar_sempty[b], 4 * C::NH);
        }
        mbar_init(&bar_quiet, 1);
        abort_flag = 0;
        fence_barrier_init();
        // Start the query tile and the first K stage right away, so that their
        // latency overlaps the tensor-memory allocation and set-up.  Issuing a
        // TMA copy takes a while and the set-up barrier waits for this thread,
        // so the producer issues the other stages after it.
        prefetch_tmap(&mQt); prefetch_tmap(&mKt); prefetch_tmap(&mQs); prefetch_tmap(&mKs);
        mbar_expect_tx(&bar_q, C::Q_BYTES);
#pragma unroll
        for (int b = 0; b < DT / 64; ++b) tma_load_3d(sQt + b * C::BLK, &mQt, &bar_q, b * 64, q0, bh, mdQt, p.st.word);
#pragma unroll
        for (int b = 0; b < DS / 64; ++b) tma_load_3d(sQs + b * C::BLK, &mQs, &bar_q, b * 64, q0, bh, mdQs, p.st.word);
        for (int kt = 0; kt < min(1, n_kt); ++kt) {
            uint8_t *st = sK + kt * C::STAGE_BYTES;
            mbar_expect_tx(&bar_kfull[kt], C::STAGE_BYTES);
#pragma unroll
            for (int b = 0; b < DT / 64; ++b)
                tma_load_3d(st + b * C::KBLK, &mKt, &bar_kfull[kt], b * 64, (kt_lo + kt) * C::BN, bkt, mdKt, p.st.word);
#pragma unroll
            for (int b = 0; b < DS / 64; ++b)
                tma_load_3d(st + C::KT_BYTES + b * C::KBLK, &mKs, &bar_kfull[kt], b * 64, (kt_lo + kt) * C::BN, bks, mdKs, p.st.word);
        }
    }
    if (warp == 1) {
        tmem_alloc(&tmem_base_sh, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base_sh;
    volatile int *abort_v = &abort_flag;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (elect_one()) {
            // Q and the first key tile were issued during set-up
            int issued = min(1, n_kt);
            for (int kt = issued; kt < n_kt; ++kt) {
                const int s = kt % C::NSTAGE, n = kt / C::NSTAGE;
                if (n > 0 && !mbar_wait(&bar_kempty[s], (n - 1) & 1, p.st, abort_v, 1)) break;
                uint8_t *st = sK + s * C::STAGE_BYTES;
                mbar_expect_tx(&bar_kfull[s], C::STAGE_BYTES);
#pragma unroll
                for (int b = 0; b < DT / 64; ++b)
                    tma_load_3d(st + b * C::KBLK, &mKt, &bar_kfull[s], b * 64, (kt_lo + kt) * C::BN, bkt, mdKt, p.st.word);
#pragma unroll
                for (int b = 0; b < DS / 64; ++b)
                    tma_load_3d(st + C::KT_BYTES + b * C::KBLK, &mKs, &bar_kfull[s], b * 64, (kt_lo + kt) * C::BN,
                                bks, mdKs, p.st.word);
                issued = kt + 1;
            }
            if (*abort_v) {
                // let copies already in flight land before the CTA's memory is released
                DevStatus quick = p.st;
                quick.budget_ns = 50000000ull;
                volatile int never = 0;
                mbar_wait(&bar_q, 0, quick, &never, 1);
                for (int kt = (issued > C::NSTAGE ? issued - C::NSTAGE : 0); kt < issued; ++kt)
                    mbar_wait(&bar_kfull[kt % C::NSTAGE], (kt / C::NSTAGE) & 1, quick, &never, 1);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        // Descriptors are built once (warp-uniform) and advanced by constant
        // offsets, so the elected thread issues one MMA every few cycles.
        const uint64_t dK0 = sw128_desc(smem_u32(sK), 16, 1024);
        if (elect_one()) {
            if (mbar_wait(&bar_qtm, 0, p.st, abort_v, 2)) {
                for (int kt = 0; kt < n_kt; ++kt) {
                    const int s = kt % C::NSTAGE, n = kt / C::NSTAGE;
                    const int buf = kt % C::NBUF, use = kt / C::NBUF;
                    if (!mbar_wait(&bar_kfull[s], n & 1, p.st, abort_v, 3)) break;
                    if (use > 0 && !mbar_wait(&bar_sempty[buf], (use - 1) & 1, p.st, abort_v, 4)) break;
                    tc_fence_after();
                    const uint64_t dKt = desc_add(dK0, s * C::STAGE_BYTES), dKs = desc_add(dKt, C::KT_BYTES);
                    const uint32_t dSt = tmem + buf * 128, dSs = dSt + 64;
#pragma unroll
                    for (int kk = 0; kk < DT / 16; ++kk) {
                        const uint32_t ok = (kk >> 2) * C::KBLK + (kk & 3) * 32;
                        mma_bf16_ts(dSt, tmem + C::TMEM_QT + kk * 8, desc_add(dKt, ok), C::IDESC, kk > 0);
                    }
#pragma unroll
                    for (int kk = 0; kk < DS / 16; ++kk) {
                        const uint32_t ok = (kk >> 2) * C::KBLK + (kk & 3) * 32;
                        mma_bf16_ts(dSs, tmem + C::TMEM_QS + kk * 8, desc_add(dKs, ok), C::IDESC, kk > 0);
                    }
                    mma_commit(&bar_sfull[buf]);
                    mma_commit(&bar_kempty[s]);
                }
            }
            mma_quiesce(&bar_quiet, p.st, 9);
        }
    } else {
        // ------------------------------------------------------------ softmax warpgroups (ping-pong)
        const int wg = (warp - 2) >> 2;
        const int par = wg & 1, half = wg >> 1;
        const int sub = warp & 3;
        const int row = sub * 32 + lane;
        const int grow = q0 + row;
        const uint32_t lane_base = tmem + ((uint32_t)(sub * 32) << 16);
        // this warp's quarter of its 32 rows of Q_t and Q_s into tensor memory
        if (mbar_wait(&bar_q, 0, p.st, abort_v, 6)) {
            tile_rows_to_tmem<DT>(lane_base + C::TMEM_QT, sQt, wg, row);
            tile_rows_to_tmem<DS>(lane_base + C::TMEM_QS, sQs, wg, row);
            tmem_st_wait();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar_qtm);
        float Mt = -INFINITY, Ms = -INFINITY, lt = 0.f, ls = 0.f, A = 0.f;
        for (int kt = par; kt < n_kt; kt += 2) {
            const int buf = kt % C::NBUF;
            const uint32_t bufc = lane_base + buf * 128;
            if (!mbar_wait(&bar_sfull[buf], (kt / C::NBUF) & 1, p.st, abort_v, 5)) break;
            tc_fence_after();
            const int k0 = (kt_lo + kt) * C::BN;
#pragma unroll
            for (int cc = 0; cc < C::CW / 32; ++cc) {
                const int c = half * (C::CW / 32) + cc;
                const int kc = k0 + c * 32;
                float ut[32], us[32];
                tmem_ld32(bufc + c * 32, ut);
                tmem_ld32(bufc + 64 + c * 32, us);
                tmem_ld_wait();
                const bool masked = (kc + 32 > nk) || (p.causal && (kc + 31 > q0 + off));
                if (masked) {
                    const int lim = p.causal ? min(nk, grow + off + 1) : nk;   // first hidden key
#pragma unroll
                    for (int k = 0; k < 32; ++k) {
                        if (kc + k >= lim) { ut[k] = -INFINITY; us[k] = -INFINITY; }
                    }
                    online_chunk_masked(ut, us, p.ct, p.cs, Mt, Ms, lt, ls, A);
                } else {
                    online_chunk_lag(ut, us, p.ct, p.cs, Mt, Ms, lt, ls, A);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar_sempty[buf]);
        }
        RowState x{Mt, Ms, lt, ls, A};
        if (NWG > 1) {
            if (wg > 0) {
                merge[wg - 1][0][row] = Mt; merge[wg - 1][1][row] = Ms; merge[wg - 1][2][row] = lt;
                merge[wg - 1][3][row] = ls; merge[wg - 1][4][row] = A;
            }
            asm volatile("bar.sync 1, %0;" ::"r"(128 * NWG) : "memory");
            if (wg == 0) {
#pragma unroll
                for (int o = 0; o < NWG - 1; ++o)
                    merge_state(x, RowState{merge[o][0][row], merge[o][1][row], merge[o][2][row], merge[o][3][row],
                                            merge[o][4][row]});
            }
        }
        if (wg == 0 && grow < p.N_Q && !*abort_v &&
            bound_ok(bh < p.BH && split < p.splits, p.st.word, kSiteRowOut)) {
            const size_t r = (size_t)bh * p.N_Q + grow;
            if (p.splits > 1) {
                const size_t rows = (size_t)p.BH * p.N_Q, fs = (size_t)p.splits * rows;
                float *q = p.part + (size_t)split * rows + r;
                q[0] = x.Mt; q[fs] = x.Ms; q[2 * fs] = x.lt; q[3 * fs] = x.ls; q[4 * fs] = x.A;
            } else {
                finish_row(x, p.kl + r, p.lse_t + r, p.lse_s + r);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

// Persistent form of streamkl_fwd_kernel: one CTA per SM works through its
// items (one 128-row query tile of one head, or one key split of it; see
// persistent_item) one after the other.  Key tiles are counted across items,
// so the K ring, the three logit buffers and their barrier phases simply
// continue from one item to the next, and tile g goes to the softmax parity
// g & 1 as in the one-item kernel.  The next item's query rows land in the
// shared-memory landing area by TMA as soon as the softmax warps have copied
// the current item's rows into tensor memory, and its first key tiles load
// while the current item is computed; what remains at an item boundary is the
// merge of the four warpgroups' row states and the copy of the next rows into
// tensor memory once the current item's last logit MMA has completed.  Set-up,
// tensor-memory allocation, the launch and the query-tile load are paid once
// per SM instead of once per query tile.
template <int DT, int DS, int NWG>
__global__ void __launch_bounds__(FwdCfg<DT, DS, NWG>::THREADS, 1)
    streamkl_fwd_persistent_kernel(const __grid_constant__ CUtensorMap mQt, const __grid_constant__ CUtensorMap mKt,
                                   const __grid_constant__ CUtensorMap mQs, const __grid_constant__ CUtensorMap mKs,
                                   const FwdParams p) {
    using C = FwdCfg<DT, DS, NWG>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sQt = smem;                  // landing area of the query rows
    uint8_t *sQs = sQt + C::QT_BYTES;
    uint8_t *sK = sQs + C::QS_BYTES;      // stage s: K_t then K_s

    __shared__ uint64_t bar_kfull[C::NSTAGE], bar_kempty[C::NSTAGE], bar_sfull[C::NBUF], bar_sempty[C::NBUF];
    __shared__ uint64_t bar_quiet;                 // the MMA thread's issued MMAs have completed
    __shared__ uint64_t bar_q;            // the item's query rows have landed
    __shared__ uint64_t bar_qfree;        // ... and been copied out of the landing area
    __shared__ uint64_t bar_qtm;          // ... and are in tensor memory
    __shared__ uint64_t bar_qtmfree;      // the item's last logit MMA has completed
    __shared__ uint32_t tmem_base_sh;
    __shared__ int abort_flag;
    // per-row states of warpgroups 1..NWG-1, double-buffered by item parity
    __shared__ float merge[2][NWG > 1 ? NWG - 1 : 1][5][128];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // tensors behind the four maps (bounds-checked build)
    const MapDims mdQt{DT, p.N_Q, p.BH}, mdQs{DS, p.N_Q, p.BH};
    const MapDims mdKt{DT, p.N_K, p.BH / p.H * p.Hkt}, mdKs{DS, p.N_K, p.BH / p.H * p.Hks};
    const int off = p.N_K - p.N_Q;
    const int n_items = p.BH * p.n_qt * p.splits;
    // item j: as block j of the one-item kernel (heaviest causal tiles first,
    // the key splits of one query tile adjacent)
    struct Item {
        int bh, split, q0, kt_lo, n_kt, bkt, bks;
    };
    auto item_geom = [&](int j, bool report) {
        Item it;
        const int lin = j / p.BH;
        it.split = lin % p.splits;
        it.bh = j % p.BH;
        it.q0 = (p.n_qt - 1 - lin / p.splits) * C::BM;
        const int nk = key_count(p.kv_len, it.bh / p.H, p.N_K, p.st.word, report);
        const int n_all = fwd_key_tiles(it.q0, p.N_Q, nk, off, p.causal, C::BN);
        it.kt_lo = (int)((long long)n_all * it.split / p.splits);
        it.n_kt = (int)((long long)n_all * (it.split + 1) / p.splits) - it.kt_lo;
        it.bkt = key_head(it.bh, p.H, p.Hkt);
        it.bks = key_head(it.bh, p.H, p.Hks);
        return it;
    };

    if (threadIdx.x == 0) {
        mbar_init(&bar_q, 1);
        mbar_init(&bar_qfree, 4 * NWG);   // every softmax warp, once it has copied its rows
        mbar_init(&bar_qtm, 4 * NWG);     // every softmax warp, once its rows are in tensor memory
        mbar_init(&bar_qtmfree, 1);
        for (int s = 0; s < C::NSTAGE; ++s) {
            mbar_init(&bar_kfull[s], 1);
            mbar_init(&bar_kempty[s], 1);
        }
        for (int b = 0; b < C::NBUF; ++b) {
            mbar_init(&bar_sfull[b], 1);
            mbar_init(&bar_sempty[b], 4 * C::NH);
        }
        mbar_init(&bar_quiet, 1);
        abort_flag = 0;
        fence_barrier_init();
        // the first item's query rows and first key tile right away (the
        // producer issues the rest after the set-up barrier)
        prefetch_tmap(&mQt); prefetch_tmap(&mKt); prefetch_tmap(&mQs); prefetch_tmap(&mKs);
        const Item it = item_geom(persistent_item(0, n_items), true);
        mbar_expect_tx(&bar_q, C::Q_BYTES);
#pragma unroll
        for (int b = 0; b < DT / 64; ++b) tma_load_3d(sQt + b * C::BLK, &mQt, &bar_q, b * 64, it.q0, it.bh, mdQt, p.st.word);
#pragma unroll
        for (int b = 0; b < DS / 64; ++b) tma_load_3d(sQs + b * C::BLK, &mQs, &bar_q, b * 64, it.q0, it.bh, mdQs, p.st.word);
        if (it.n_kt > 0) {
            mbar_expect_tx(&bar_kfull[0], C::STAGE_BYTES);
#pragma unroll
            for (int b = 0; b < DT / 64; ++b)
                tma_load_3d(sK + b * C::KBLK, &mKt, &bar_kfull[0], b * 64, it.kt_lo * C::BN, it.bkt, mdKt, p.st.word);
#pragma unroll
            for (int b = 0; b < DS / 64; ++b)
                tma_load_3d(sK + C::KT_BYTES + b * C::KBLK, &mKs, &bar_kfull[0], b * 64, it.kt_lo * C::BN, it.bks,
                            mdKs, p.st.word);
        }
    }
    if (warp == 1) {
        tmem_alloc(&tmem_base_sh, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base_sh;
    volatile int *abort_v = &abort_flag;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (elect_one()) {
            int g = 0, issued = 0, q_issued = 1;      // key tiles issued (counted across items), query loads
            bool ok = true;
            for (int r = 0, itn = 0; ok; ++r, ++itn) {
                const int j = persistent_item(r, n_items);
                if (j < 0) break;
                const Item it = item_geom(j, false);
                if (r > 0) {
                    // the landing area is free once the previous item's rows are copied out
                    if (!mbar_wait(&bar_qfree, (itn - 1) & 1, p.st, abort_v, 7)) break;
                    mbar_expect_tx(&bar_q, C::Q_BYTES);
#pragma unroll
                    for (int b = 0; b < DT / 64; ++b)
                        tma_load_3d(sQt + b * C::BLK, &mQt, &bar_q, b * 64, it.q0, it.bh, mdQt, p.st.word);
#pragma unroll
                    for (int b = 0; b < DS / 64; ++b)
                        tma_load_3d(sQs + b * C::BLK, &mQs, &bar_q, b * 64, it.q0, it.bh, mdQs, p.st.word);
                    ++q_issued;
                }
                for (int kt = 0; kt < it.n_kt; ++kt, ++g) {
                    if (r == 0 && kt == 0) {            // issued during set-up
                        issued = 1;
                        continue;
                    }
                    const int s = g % C::NSTAGE, n = g / C::NSTAGE;
                    if (n > 0 && !mbar_wait(&bar_kempty[s], (n - 1) & 1, p.st, abort_v, 1)) { ok = false; break; }
                    uint8_t *st = sK + s * C::STAGE_BYTES;
                    mbar_expect_tx(&bar_kfull[s], C::STAGE_BYTES);
#pragma unroll
                    for (int b = 0; b < DT / 64; ++b)
                        tma_load_3d(st + b * C::KBLK, &mKt, &bar_kfull[s], b * 64, (it.kt_lo + kt) * C::BN, it.bkt,
                                    mdKt, p.st.word);
#pragma unroll
                    for (int b = 0; b < DS / 64; ++b)
                        tma_load_3d(st + C::KT_BYTES + b * C::KBLK, &mKs, &bar_kfull[s], b * 64,
                                    (it.kt_lo + kt) * C::BN, it.bks, mdKs, p.st.word);
                    issued = g + 1;
                }
            }
            if (*abort_v) {
                // let copies already in flight land before the CTA's memory is released
                DevStatus quick = p.st;
                quick.budget_ns = 50000000ull;
                volatile int never = 0;
                mbar_wait(&bar_q, (q_issued - 1) & 1, quick, &never, 1);
                for (int t = (issued > C::NSTAGE ? issued - C::NSTAGE : 0); t < issued; ++t)
                    mbar_wait(&bar_kfull[t % C::NSTAGE], (t / C::NSTAGE) & 1, quick, &never, 1);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        const uint64_t dK0 = sw128_desc(smem_u32(sK), 16, 1024);
        if (elect_one()) {
            int g = 0;
            bool ok = true;
            for (int r = 0, itn = 0; ok; ++r, ++itn) {
                const int j = persistent_item(r, n_items);
                if (j < 0) break;
                const Item it = item_geom(j, false);
                if (!mbar_wait(&bar_qtm, itn & 1, p.st, abort_v, 2)) break;
                for (int kt = 0; kt < it.n_kt; ++kt, ++g) {
                    const int s = g % C::NSTAGE, n = g / C::NSTAGE;
                    const int buf = g % C::NBUF, use = g / C::NBUF;
                    if (!mbar_wait(&bar_kfull[s], n & 1, p.st, abort_v, 3)) { ok = false; break; }
                    if (use > 0 && !mbar_wait(&bar_sempty[buf], (use - 1) & 1, p.st, abort_v, 4)) { ok = false; break; }
                    tc_fence_after();
                    const uint64_t dKt = desc_add(dK0, s * C::STAGE_BYTES), dKs = desc_add(dKt, C::KT_BYTES);
                    const uint32_t dSt = tmem + buf * 128, dSs = dSt + 64;
#pragma unroll
                    for (int kk = 0; kk < DT / 16; ++kk) {
                        const uint32_t ok2 = (kk >> 2) * C::KBLK + (kk & 3) * 32;
                        mma_bf16_ts(dSt, tmem + C::TMEM_QT + kk * 8, desc_add(dKt, ok2), C::IDESC, kk > 0);
                    }
#pragma unroll
                    for (int kk = 0; kk < DS / 16; ++kk) {
                        const uint32_t ok2 = (kk >> 2) * C::KBLK + (kk & 3) * 32;
                        mma_bf16_ts(dSs, tmem + C::TMEM_QS + kk * 8, desc_add(dKs, ok2), C::IDESC, kk > 0);
                    }
                    mma_commit(&bar_sfull[buf]);
                    mma_commit(&bar_kempty[s]);
                }
                if (!ok) break;
                mma_commit(&bar_qtmfree);       // the item's query rows in tensor memory may go
            }
            mma_quiesce(&bar_quiet, p.st, 9);
        }
    } else {
        // ------------------------------------------------------------ softmax warpgroups (ping-pong)
        const int wg = (warp - 2) >> 2;
        const int par = wg & 1, half = wg >> 1;
        const int sub = warp & 3;
        const int row = sub * 32 + lane;
        const uint32_t lane_base = tmem + ((uint32_t)(sub * 32) << 16);
        int g0 = 0;
        for (int r = 0, itn = 0;; ++r, ++itn) {
            const int j = persistent_item(r, n_items);
            if (j < 0) break;
            const Item it = item_geom(j, false);
            const int grow = it.q0 + row;
            // this warp's quarter of its 32 rows of Q_t and Q_s into tensor memory,
            // once they have landed and the previous item's logit MMAs are done.
            // A wait that gives up ends the item's work but not its merge
            // barrier, which every softmax warp reaches (the exit is decided there).
            bool ok = mbar_wait(&bar_q, itn & 1, p.st, abort_v, 6) &&
                      (itn == 0 || mbar_wait(&bar_qtmfree, (itn - 1) & 1, p.st, abort_v, 8));
            if (ok) {
                tc_fence_after();
                tile_rows_to_tmem<DT>(lane_base + C::TMEM_QT, sQt, wg, row);
                tile_rows_to_tmem<DS>(lane_base + C::TMEM_QS, sQs, wg, row);
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(&bar_qfree);
                    mbar_arrive(&bar_qtm);
                }
            }
            float Mt = -INFINITY, Ms = -INFINITY, lt = 0.f, ls = 0.f, A = 0.f;
            const int nk = key_count(p.kv_len, it.bh / p.H, p.N_K, nullptr, false);
            for (int kt = 0; ok && kt < it.n_kt; ++kt) {
                const int g = g0 + kt;
                if ((g & 1) != par) continue;
                const int buf = g % C::NBUF;
                const uint32_t bufc = lane_base + buf * 128;
                if (!mbar_wait(&bar_sfull[buf], (g / C::NBUF) & 1, p.st, abort_v, 5)) { ok = false; break; }
                tc_fence_after();
                const int k0 = (it.kt_lo + kt) * C::BN;
#pragma unroll
                for (int cc = 0; cc < C::CW / 32; ++cc) {
                    const int c = half * (C::CW / 32) + cc;
                    const int kc = k0 + c * 32;
                    float ut[32], us[32];
                    tmem_ld32(bufc + c * 32, ut);
                    tmem_ld32(bufc + 64 + c * 32, us);
                    tmem_ld_wait();
                    const bool masked = (kc + 32 > nk) || (p.causal && (kc + 31 > it.q0 + off));
                    if (masked) {
                        const int lim = p.causal ? min(nk, grow + off + 1) : nk;   // first hidden key
#pragma unroll
                        for (int k = 0; k < 32; ++k) {
                            if (kc + k >= lim) { ut[k] = -INFINITY; us[k] = -INFINITY; }
                        }
                        online_chunk_masked(ut, us, p.ct, p.cs, Mt, Ms, lt, ls, A);
                    } else {
                        online_chunk_lag(ut, us, p.ct, p.cs, Mt, Ms, lt, ls, A);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bar_sempty[buf]);
            }
            g0 += it.n_kt;
            // merge the four warpgroups' states (double-buffered by item parity,
            // so one barrier per item suffices) and write the row outputs; the
            // barrier also tells every softmax warp alike whether to stop
            RowState x{Mt, Ms, lt, ls, A};
            float (*mg)[5][128] = merge[itn & 1];
            if (wg > 0) {
                mg[wg - 1][0][row] = Mt; mg[wg - 1][1][row] = Ms; mg[wg - 1][2][row] = lt;
                mg[wg - 1][3][row] = ls; mg[wg - 1][4][row] = A;
            }
            if (bar_sync_or(1, 128 * NWG, !ok || *abort_v)) break;
            if (wg == 0) {
#pragma unroll
                for (int o = 0; o < NWG - 1; ++o)
                    merge_state(x, RowState{mg[o][0][row], mg[o][1][row], mg[o][2][row], mg[o][3][row], mg[o][4][row]});
                if (grow < p.N_Q && bound_ok(it.bh < p.BH && it.split < p.splits, p.st.word, kSiteRowOut)) {
                    const size_t rr = (size_t)it.bh * p.N_Q + grow;
                    if (p.splits > 1) {
                        const size_t rows = (size_t)p.BH * p.N_Q, fs = (size_t)p.splits * rows;
                        float *q = p.part + (size_t)it.split * rows + rr;
                        q[0] = x.Mt; q[fs] = x.Ms; q[2 * fs] = x.lt; q[3 * fs] = x.ls; q[4 * fs] = x.A;
                    } else {
                        finish_row(x, p.kl + rr, p.lse_t + rr, p.lse_s + rr);
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

// Combines the partial states of the key splits of every row, in split
// order (so the result is the same run to run), and writes the row outputs.
__global__ void __launch_bounds__(256) streamkl_fwd_merge_kernel(const float *__restrict__ part, int splits,
                                                                 long long rows, float *__restrict__ kl,
                                                                 float *__restrict__ lse_t,
                                                                 float *__restrict__ lse_s) {
    const long long r = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (r >= rows) return;
    const long long fs = (long long)splits * rows;
    RowState x{-INFINITY, -INFINITY, 0.f, 0.f, 0.f};
    for (int s = 0; s < splits; ++s) {
        const float *q = part + (long long)s * rows + r;
        merge_state(x, RowState{q[0], q[fs], q[2 * fs], q[3 * fs], q[4 * fs]});
    }
    finish_row(x, kl + r, lse_t + r, lse_s + r);
}

// Deterministic reduction of n per-row values: out = (sum / div) * mul (the
// mean with div = n, mul = 1).  One cluster of kMeanCtas CTAs (a single CTA
// cannot keep enough loads in flight to read a large array quickly): CTA r
// sums the r-th of kMeanCtas fixed slices, each thread a fixed strided subset
// in fp64 (16-byte loads, eight in flight per thread when the array is 16-byte
// aligned), then a fixed-shape tree (warp shuffles, then one warp over the
// warp sums); CTA 0 adds the kMeanCtas slice totals in rank order, read from
// the other CTAs' shared memory.  The order of additions depends only on n
// (and the alignment), so the result is the same run to run.
constexpr int kMeanThreads = 1024, kMeanCtas = 8;

__device__ __forceinline__ unsigned cluster_rank() {
    unsigned r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// every thread of every CTA of the cluster; orders shared-memory writes
// before the barrier with reads after it, across the cluster
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// a double in the shared memory of CTA `rank` of this cluster, at the address
// `p` has in this CTA
__device__ __forceinline__ double ld_cluster_f64(const double *p, unsigned rank) {
    uint32_t ra;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(smem_u32(p)), "r"(rank));
    double v;
    asm volatile("ld.shared::cluster.f64 %0, [%1];" : "=d"(v) : "r"(ra) : "memory");
    return v;
}

__global__ void __cluster_dims__(kMeanCtas, 1, 1) __launch_bounds__(kMeanThreads)
    streamkl_mean_kernel(const float *__restrict__ v, long long n, double div, double mul, float *__restrict__ out) {
    __shared__ double red[kMeanThreads / 32];
    __shared__ double part;
    const unsigned rank = cluster_rank();
    double s = 0.0;
    if ((reinterpret_cast<uintptr_t>(v) & 15) == 0) {
        // 16-byte groups [g0, g1) of this slice; the last slice also takes the
        // elements past the last whole group
        const float4 *v4 = reinterpret_cast<const float4 *>(v);
        const long long n4 = n >> 2;
        const long long g0 = n4 * rank / kMeanCtas, g1 = n4 * (rank + 1) / kMeanCtas;
        constexpr int U = 8;
        long long k = g0 + threadIdx.x;
        for (; k + (long long)(U - 1) * kMeanThreads < g1; k += (long long)U * kMeanThreads) {
            float4 x[U];
#pragma unroll
            for (int u = 0; u < U; ++u) x[u] = __ldg(v4 + k + (long long)u * kMeanThreads);
#pragma unroll
            for (int u = 0; u < U; ++u) s += ((double)x[u].x + (double)x[u].y) + ((double)x[u].z + (double)x[u].w);
        }
        for (; k < g1; k += kMeanThreads) {
            const float4 x = __ldg(v4 + k);
            s += ((double)x.x + (double)x.y) + ((double)x.z + (double)x.w);
        }
        if (rank == kMeanCtas - 1)
            for (long long e = (n4 << 2) + threadIdx.x; e < n; e += kMeanThreads) s += (double)v[e];
    } else {
        const long long e0 = n * rank / kMeanCtas, e1 = n * (rank + 1) / kMeanCtas;
        for (long long e = e0 + threadIdx.x; e < e1; e += kMeanThreads) s += (double)v[e];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
    __syncthreads();
    if (threadIdx.x < 32) {
        s = red[threadIdx.x];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if (threadIdx.x == 0) part = s;
    }
    cluster_sync();
    if (rank == 0 && threadIdx.x == 0) {
        double total = 0.0;
        for (unsigned r = 0; r < kMeanCtas; ++r) total += ld_cluster_f64(&part, r);
        *out = n > 0 ? (float)((total / div) * mul) : 0.f;
    }
    cluster_sync();                                // CTA 0 has read every slice total
}

}  // namespace skl
