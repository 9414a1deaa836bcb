// bwd.cuh — recompute backward of the attention-distillation KL divergence.
//
// Source: "StreamKL: Fast and Memory-Efficient KL Divergence for Boosting
// Attention Distillation", abstract — the backward recomputes the attention
// probabilities tile by tile instead of storing quadratic intermediates.
//
// With g_i the upstream gradient of row i and, in log2 units,
//   a_t = y_t - L_t = (s_t - LSE_t) log2(e),   a_s = (s_s - LSE_s) log2(e),
//   P = 2^a_t,  Q = 2^a_s,
// the score gradients are
//   dS_s = g (Q - P)
//   dS_t = g P (ln P - ln Q - KL) = ln2 * [ g P (a_t - a_s - KL log2(e)) ]
// and the ln2 of the teacher side is folded into its output scale.
//
// Two kernels, each owning one side of the contraction so that every output
// accumulates in tensor memory and is written exactly once (no atomics, and a
// deterministic result):
//   streamkl_bwd_dkv_kernel  CTA = 128 keys of one head; loops over 64-query
//       tiles: S^T = K Q^T for teacher and student (tcgen05, TMEM), dS^T in
//       bf16 to shared memory, dK += dS^T Q accumulated in TMEM.  Thread =
//       key row; per-query constants come from a small shared-memory table
//       that the producer warp fills next to each TMA tile.  Two gradient
//       warpgroups split the 64 columns of a tile (32 each).
//   streamkl_bwd_dq_kernel   CTA = 128 queries of one head; loops over 64-key
//       tiles: S = Q K^T, dS in bf16 to shared memory, dQ += dS K in TMEM.
//       Thread = query row; per-row constants live in registers; two
//       gradient warpgroups split the 64 columns of a tile.
// Both recompute S: that costs one extra pair of QK^T products per element
// but removes the fp32 read-modify-write traffic a single kernel would need
// for the side it does not own.
#pragma once

#include "sm100.cuh"

namespace skl {

struct BwdParams {
    int BH, N_Q, N_K, causal, n_tiles;
    float ct, cs;                 // scale * log2(e)
    float out_t, out_s;           // output scales: scale_t * ln2 (teacher), scale_s (student)
    const float *kl, *lse_t, *lse_s, *dkl;
    float g_const;                // g when dkl == nullptr
    float *dq_s, *dq_t, *dk_s, *dk_t;
    DevStatus st;
};

constexpr float kLog2eF = 1.4426950408889634074f;

// dS for two adjacent elements, packed as bf16x2.
template <bool TEACHER, bool MASKED>
__device__ __forceinline__ void ds_pair(float ut0, float ut1, float us0, float us1, float ct, float cs, float Lt,
                                        float Ls, float g, float KL2, bool vis0, bool vis1, uint32_t &ps,
                                        uint32_t &pt) {
    const float at0 = fmaf(ut0, ct, -Lt), at1 = fmaf(ut1, ct, -Lt);
    const float as0 = fmaf(us0, cs, -Ls), as1 = fmaf(us1, cs, -Ls);
    float P0 = ex2(at0), P1 = ex2(at1);
    float Q0 = ex2(as0), Q1 = ex2(as1);
    if (MASKED) {
        P0 = vis0 ? P0 : 0.f; Q0 = vis0 ? Q0 : 0.f;
        P1 = vis1 ? P1 : 0.f; Q1 = vis1 ? Q1 : 0.f;
    }
    ps = pack_bf16(g * (Q0 - P0), g * (Q1 - P1));
    if (TEACHER) {
        const float gP0 = g * P0, gP1 = g * P1;
        pt = pack_bf16(gP0 * ((at0 - as0) - KL2), gP1 * ((at1 - as1) - KL2));
    }
}

// Stores 64 bf16 (32 packed pairs) as row `row` of a [rows][64] 128B-swizzled tile.
__device__ __forceinline__ void store_row64(uint8_t *tile, int row, const uint32_t (&v)[32]) {
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        const uint32_t off = (uint32_t)row * 128u + ((uint32_t)(c ^ (row & 7)) << 4);
        *reinterpret_cast<uint4 *>(tile + off) = make_uint4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
    }
}

// Stores 32 bf16 (16 packed pairs) as 16-byte chunks chunk0..chunk0+3 of row `row`
// of a [rows][64] 128B-swizzled tile.
__device__ __forceinline__ void store_row32(uint8_t *tile, int row, int chunk0, const uint32_t (&v)[16]) {
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const uint32_t off = (uint32_t)row * 128u + ((uint32_t)((chunk0 + c) ^ (row & 7)) << 4);
        *reinterpret_cast<uint4 *>(tile + off) = make_uint4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
    }
}

// Reads `ncols` fp32 accumulator columns of this thread's TMEM lane, scales them
// and writes them to dst (one row, contiguous) if `store`.
template <int NCOLS>
__device__ __forceinline__ void drain_row(uint32_t taddr, float scale, float *dst, bool store) {
#pragma unroll 1
    for (int c = 0; c < NCOLS / 32; ++c) {
        float v[32];
        tmem_ld32(taddr + c * 32, v);
        tmem_ld_wait();
        if (store) {
            float4 *d4 = reinterpret_cast<float4 *>(dst + c * 32);
#pragma unroll
            for (int k = 0; k < 8; ++k)
                d4[k] = make_float4(v[4 * k] * scale, v[4 * k + 1] * scale, v[4 * k + 2] * scale,
                                    v[4 * k + 3] * scale);
        }
    }
}

// ============================================================================ dK kernel
constexpr int kBwdWarpgroups = 2;    // gradient warpgroups per CTA; each takes 32 columns of a tile

template <int DT, int DS, bool TEACHER>
struct DkvCfg {
    static constexpr int BN = 128, BM = 64;       // keys per CTA, queries per tile
    static constexpr int KBLK = 128 * 128;         // [128 rows][64] bf16 box
    static constexpr int QBLK = 64 * 128;          // [64 rows][64] bf16 box
    static constexpr int KT_BYTES = BN * DT * 2, KS_BYTES = BN * DS * 2;
    static constexpr int QT_BYTES = BM * DT * 2, QS_BYTES = BM * DS * 2;
    static constexpr int CONST_BYTES = BM * 16;   // float4 per query
    static constexpr int STAGE_TMA = QT_BYTES + QS_BYTES;
    static constexpr int STAGE_BYTES = STAGE_TMA + CONST_BYTES;
    static constexpr int DSB = BN * BM * 2;        // one dS^T tile, bf16
    static constexpr int DS_BYTES = DSB * (TEACHER ? 2 : 1);
    static constexpr int FIXED = KT_BYTES + KS_BYTES + DS_BYTES;
    static constexpr int NS_RAW = (210 * 1024 - FIXED) / STAGE_BYTES;
    static constexpr int NSTAGE = NS_RAW < 2 ? 2 : (NS_RAW > 4 ? 4 : NS_RAW);
    static constexpr int SMEM = FIXED + NSTAGE * STAGE_BYTES + 1024;
    static constexpr int NWG = kBwdWarpgroups;
    static constexpr int THREADS = 64 + 128 * NWG;
    static constexpr uint32_t IDESC_S = idesc_bf16(128, BM, 0, 0);
    static constexpr uint32_t IDESC_KS = idesc_bf16(128, DS, 0, 1);
    static constexpr uint32_t IDESC_KT = idesc_bf16(128, DT, 0, 1);
    static constexpr uint32_t TMEM_DKS = 256, TMEM_DKT = 256 + DS;
};

template <int DT, int DS, bool TEACHER>
__global__ void __launch_bounds__(DkvCfg<DT, DS, TEACHER>::THREADS, 1)
    streamkl_bwd_dkv_kernel(const __grid_constant__ CUtensorMap mQt, const __grid_constant__ CUtensorMap mKt,
                            const __grid_constant__ CUtensorMap mQs, const __grid_constant__ CUtensorMap mKs,
                            const BwdParams p) {
    using C = DkvCfg<DT, DS, TEACHER>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sKt = smem;
    uint8_t *sKs = sKt + C::KT_BYTES;
    uint8_t *sDss = sKs + C::KS_BYTES;             // dS_s^T  [128 keys][64 queries]
    uint8_t *sDst = sDss + C::DSB;                 // dS_t^T  (teacher)
    uint8_t *sQ = sKs + C::KS_BYTES + C::DS_BYTES; // stages: Q_t, Q_s, constants

    __shared__ uint64_t bar_k, bar_qfull[C::NSTAGE], bar_qempty[C::NSTAGE], bar_sfull[2], bar_sempty[2];
    __shared__ uint64_t bar_dsfull, bar_dsempty, bar_done;
    __shared__ uint32_t tmem_base_sh;
    __shared__ int abort_flag;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int kt_idx = (int)(blockIdx.x / p.BH);   // low key tiles see the most queries: run them first
    const int bh = (int)(blockIdx.x % p.BH);
    const int k0 = kt_idx * C::BN;
    const int off = p.N_K - p.N_Q;
    const int n_qt_all = (p.N_Q + C::BM - 1) / C::BM;
    const int first_qt = p.causal ? max(0, k0 - off) / C::BM : 0;
    const int n_qt = max(0, n_qt_all - first_qt);

    if (threadIdx.x == 0) {
        mbar_init(&bar_k, 1);
        for (int s = 0; s < C::NSTAGE; ++s) {
            mbar_init(&bar_qfull[s], 1 + 32);      // TMA expect_tx + every producer lane (constants)
            mbar_init(&bar_qempty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bar_sfull[b], 1);
            mbar_init(&bar_sempty[b], 4 * C::NWG);
        }
        mbar_init(&bar_dsfull, 4 * C::NWG);
        mbar_init(&bar_dsempty, 1);
        mbar_init(&bar_done, 1);
        abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(&tmem_base_sh, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base_sh;
    volatile int *abort_v = &abort_flag;

    if (warp == 0) {
        // ------------------------------------------------------------ producer (TMA + per-query constants)
        if (lane == 0) {
            prefetch_tmap(&mQt); prefetch_tmap(&mKt); prefetch_tmap(&mQs); prefetch_tmap(&mKs);
            mbar_expect_tx(&bar_k, C::KT_BYTES + C::KS_BYTES);
#pragma unroll
            for (int b = 0; b < DT / 64; ++b) tma_load_3d(sKt + b * C::KBLK, &mKt, &bar_k, b * 64, k0, bh);
#pragma unroll
            for (int b = 0; b < DS / 64; ++b) tma_load_3d(sKs + b * C::KBLK, &mKs, &bar_k, b * 64, k0, bh);
        }
        int issued = 0;
        for (int t = 0; t < n_qt; ++t) {
            const int s = t % C::NSTAGE, n = t / C::NSTAGE;
            const int q0 = (first_qt + t) * C::BM;
            if (n > 0 && !mbar_wait(&bar_qempty[s], (n - 1) & 1, p.st, abort_v, 11)) break;
            uint8_t *st = sQ + s * C::STAGE_BYTES;
            if (lane == 0) {
                mbar_expect_tx(&bar_qfull[s], C::STAGE_TMA);
#pragma unroll
                for (int b = 0; b < DT / 64; ++b)
                    tma_load_3d(st + b * C::QBLK, &mQt, &bar_qfull[s], b * 64, q0, bh);
#pragma unroll
                for (int b = 0; b < DS / 64; ++b)
                    tma_load_3d(st + C::QT_BYTES + b * C::QBLK, &mQs, &bar_qfull[s], b * 64, q0, bh);
            }
            float4 *cst = reinterpret_cast<float4 *>(st + C::STAGE_TMA);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int q = lane + 32 * h;
                const int i = q0 + q;
                float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
                if (i < p.N_Q) {
                    const size_t r = (size_t)bh * p.N_Q + i;
                    v.x = p.lse_t[r] * kLog2eF;
                    v.y = p.lse_s[r] * kLog2eF;
                    v.z = p.dkl ? p.dkl[r] : p.g_const;
                    v.w = p.kl[r] * kLog2eF;
                }
                cst[q] = v;
            }
            mbar_arrive(&bar_qfull[s]);
            issued = t + 1;
        }
        if (*abort_v && lane == 0) {
            DevStatus quick = p.st;
            quick.budget_ns = 50000000ull;
            volatile int never = 0;
            mbar_wait(&bar_k, 0, quick, &never, 11);
            for (int t = (issued > C::NSTAGE ? issued - C::NSTAGE : 0); t < issued; ++t)
                mbar_wait(&bar_qfull[t % C::NSTAGE], (t / C::NSTAGE) & 1, quick, &never, 11);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (elect_one()) {
            const uint32_t aKt = smem_u32(sKt), aKs = smem_u32(sKs);
            const uint32_t aDss = smem_u32(sDss), aDst = smem_u32(sDst);
            auto issue_s = [&](int t) -> bool {
                const int s = t % C::NSTAGE, n = t / C::NSTAGE, buf = t & 1, use = t >> 1;
                if (!mbar_wait(&bar_qfull[s], n & 1, p.st, abort_v, 12)) return false;
                if (use > 0 && !mbar_wait(&bar_sempty[buf], (use - 1) & 1, p.st, abort_v, 13)) return false;
                tc_fence_after();
                const uint32_t aQt = smem_u32(sQ + s * C::STAGE_BYTES), aQs = aQt + C::QT_BYTES;
#pragma unroll
                for (int kk = 0; kk < DT / 16; ++kk)
                    mma_bf16_ss(tmem + buf * 128, sw128_desc(aKt + (kk >> 2) * C::KBLK + (kk & 3) * 32, 16, 1024),
                                sw128_desc(aQt + (kk >> 2) * C::QBLK + (kk & 3) * 32, 16, 1024), C::IDESC_S, kk > 0);
#pragma unroll
                for (int kk = 0; kk < DS / 16; ++kk)
                    mma_bf16_ss(tmem + buf * 128 + 64,
                                sw128_desc(aKs + (kk >> 2) * C::KBLK + (kk & 3) * 32, 16, 1024),
                                sw128_desc(aQs + (kk >> 2) * C::QBLK + (kk & 3) * 32, 16, 1024), C::IDESC_S, kk > 0);
                mma_commit(&bar_sfull[buf]);
                return true;
            };
            bool ok = mbar_wait(&bar_k, 0, p.st, abort_v, 14);
            if (ok && n_qt > 0) ok = issue_s(0);
            for (int t = 0; ok && t < n_qt; ++t) {
                if (t + 1 < n_qt && !issue_s(t + 1)) break;
                if (!mbar_wait(&bar_dsfull, t & 1, p.st, abort_v, 15)) break;
                tc_fence_after();
                const int s = t % C::NSTAGE;
                const uint32_t aQt = smem_u32(sQ + s * C::STAGE_BYTES), aQs = aQt + C::QT_BYTES;
#pragma unroll
                for (int ks = 0; ks < C::BM / 16; ++ks)
                    mma_bf16_ss(tmem + C::TMEM_DKS, sw128_desc(aDss + ks * 32, 16, 1024),
                                sw128_desc(aQs + ks * 2048, C::QBLK, 1024), C::IDESC_KS, (t > 0 || ks > 0));
                if (TEACHER) {
#pragma unroll
                    for (int ks = 0; ks < C::BM / 16; ++ks)
                        mma_bf16_ss(tmem + C::TMEM_DKT, sw128_desc(aDst + ks * 32, 16, 1024),
                                    sw128_desc(aQt + ks * 2048, C::QBLK, 1024), C::IDESC_KT, (t > 0 || ks > 0));
                }
                mma_commit(&bar_dsempty);
                mma_commit(&bar_qempty[s]);
            }
            mma_commit(&bar_done);
        }
    } else {
        // ------------------------------------------------------------ gradient warpgroups (thread = key)
        // Warpgroup wg handles query columns [32 wg, 32 wg + 32) of every tile and
        // drains its share of the dK columns at the end.
        const int wg = (warp - 2) >> 2;
        const int sub = warp & 3;
        const int row = sub * 32 + lane;
        const int gk = k0 + row;
        const int c0 = wg * 32;
        const uint32_t lane_base = tmem + ((uint32_t)(sub * 32) << 16);
        bool ok = true;
        for (int t = 0; t < n_qt; ++t) {
            const int s = t % C::NSTAGE, n = t / C::NSTAGE, buf = t & 1, use = t >> 1;
            const int q0 = (first_qt + t) * C::BM;
            if (!mbar_wait(&bar_sfull[buf], use & 1, p.st, abort_v, 16) ||
                !mbar_wait(&bar_qfull[s], n & 1, p.st, abort_v, 17)) { ok = false; break; }
            tc_fence_after();
            const float4 *cst = reinterpret_cast<const float4 *>(sQ + s * C::STAGE_BYTES + C::STAGE_TMA) + c0;
            const bool masked = p.causal && (k0 + C::BN - 1 > q0 + c0 + off);
            const int qmin = gk - off - (q0 + c0);   // first visible query column of this warpgroup (causal)
            uint32_t ps[16], pt[16];
            {
                float ut[32], us[32];
                tmem_ld32(lane_base + buf * 128 + c0, ut);
                tmem_ld32(lane_base + buf * 128 + 64 + c0, us);
                tmem_ld_wait();
#pragma unroll
                for (int k = 0; k < 32; k += 2) {
                    const float4 e0 = cst[k], e1 = cst[k + 1];
                    float at0 = fmaf(ut[k], p.ct, -e0.x), at1 = fmaf(ut[k + 1], p.ct, -e1.x);
                    float as0 = fmaf(us[k], p.cs, -e0.y), as1 = fmaf(us[k + 1], p.cs, -e1.y);
                    float P0 = ex2(at0), P1 = ex2(at1), Q0 = ex2(as0), Q1 = ex2(as1);
                    if (masked) {
                        if (k < qmin) { P0 = 0.f; Q0 = 0.f; }
                        if (k + 1 < qmin) { P1 = 0.f; Q1 = 0.f; }
                    }
                    ps[k >> 1] = pack_bf16(e0.z * (Q0 - P0), e1.z * (Q1 - P1));
                    if (TEACHER)
                        pt[k >> 1] = pack_bf16((e0.z * P0) * ((at0 - as0) - e0.w), (e1.z * P1) * ((at1 - as1) - e1.w));
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar_sempty[buf]);
            if (t > 0 && !mbar_wait(&bar_dsempty, (t - 1) & 1, p.st, abort_v, 18)) { ok = false; break; }
            store_row32(sDss, row, wg * 4, ps);
            if (TEACHER) store_row32(sDst, row, wg * 4, pt);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar_dsfull);
        }
        if (ok && n_qt > 0 && mbar_wait(&bar_done, 0, p.st, abort_v, 19)) {
            tc_fence_after();
            const bool store = gk < p.N_K;
            const size_t r = (size_t)bh * p.N_K + (store ? gk : 0);
            constexpr int HS = DS / C::NWG, HT = DT / C::NWG;
            drain_row<HS>(lane_base + C::TMEM_DKS + wg * HS, p.out_s, p.dk_s + r * DS + wg * HS, store);
            if (TEACHER) drain_row<HT>(lane_base + C::TMEM_DKT + wg * HT, p.out_t, p.dk_t + r * DT + wg * HT, store);
        } else if (n_qt == 0 && gk < p.N_K && wg == 0) {
            const size_t r = (size_t)bh * p.N_K + gk;
            for (int c = 0; c < DS; ++c) p.dk_s[r * DS + c] = 0.f;
            if (TEACHER) for (int c = 0; c < DT; ++c) p.dk_t[r * DT + c] = 0.f;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ============================================================================ dQ kernel
template <int DT, int DS, bool TEACHER>
struct DqCfg {
    static constexpr int BM = 128, BN = 64;       // queries per CTA, keys per tile
    static constexpr int QBLK = 128 * 128;         // [128 rows][64] bf16 box
    static constexpr int KBLK = 64 * 128;          // [64 rows][64] bf16 box
    static constexpr int QT_BYTES = BM * DT * 2, QS_BYTES = BM * DS * 2;
    static constexpr int KT_BYTES = BN * DT * 2, KS_BYTES = BN * DS * 2;
    static constexpr int STAGE_BYTES = KT_BYTES + KS_BYTES;
    static constexpr int DSB = BM * BN * 2;
    static constexpr int DS_BYTES = DSB * (TEACHER ? 2 : 1);
    static constexpr int FIXED = QT_BYTES + QS_BYTES + DS_BYTES;
    static constexpr int NS_RAW = (210 * 1024 - FIXED) / STAGE_BYTES;
    static constexpr int NSTAGE = NS_RAW < 2 ? 2 : (NS_RAW > 4 ? 4 : NS_RAW);
    static constexpr int SMEM = FIXED + NSTAGE * STAGE_BYTES + 1024;
    static constexpr int NWG = kBwdWarpgroups;
    static constexpr int THREADS = 64 + 128 * NWG;
    static constexpr uint32_t IDESC_S = idesc_bf16(128, BN, 0, 0);
    static constexpr uint32_t IDESC_QS = idesc_bf16(128, DS, 0, 1);
    static constexpr uint32_t IDESC_QT = idesc_bf16(128, DT, 0, 1);
    static constexpr uint32_t TMEM_DQS = 256, TMEM_DQT = 256 + DS;
};

template <int DT, int DS, bool TEACHER>
__global__ void __launch_bounds__(DqCfg<DT, DS, TEACHER>::THREADS, 1)
    streamkl_bwd_dq_kernel(const __grid_constant__ CUtensorMap mQt, const __grid_constant__ CUtensorMap mKt,
                           const __grid_constant__ CUtensorMap mQs, const __grid_constant__ CUtensorMap mKs,
                           const BwdParams p) {
    using C = DqCfg<DT, DS, TEACHER>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sQt = smem;
    uint8_t *sQs = sQt + C::QT_BYTES;
    uint8_t *sDss = sQs + C::QS_BYTES;             // dS_s [128 queries][64 keys]
    uint8_t *sDst = sDss + C::DSB;
    uint8_t *sK = sQs + C::QS_BYTES + C::DS_BYTES; // stages: K_t, K_s

    __shared__ uint64_t bar_q, bar_kfull[C::NSTAGE], bar_kempty[C::NSTAGE], bar_sfull[2], bar_sempty[2];
    __shared__ uint64_t bar_dsfull, bar_dsempty, bar_done;
    __shared__ uint32_t tmem_base_sh;
    __shared__ int abort_flag;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int qt_idx = p.n_tiles - 1 - (int)(blockIdx.x / p.BH);
    const int bh = (int)(blockIdx.x % p.BH);
    const int q0 = qt_idx * C::BM;
    const int off = p.N_K - p.N_Q;
    int kend = p.N_K;
    if (p.causal) kend = min(p.N_K, min(q0 + C::BM - 1, p.N_Q - 1) + off + 1);
    const int n_kt = (kend + C::BN - 1) / C::BN;

    if (threadIdx.x == 0) {
        mbar_init(&bar_q, 1);
        for (int s = 0; s < C::NSTAGE; ++s) {
            mbar_init(&bar_kfull[s], 1);
            mbar_init(&bar_kempty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bar_sfull[b], 1);
            mbar_init(&bar_sempty[b], 4 * C::NWG);
        }
        mbar_init(&bar_dsfull, 4 * C::NWG);
        mbar_init(&bar_dsempty, 1);
        mbar_init(&bar_done, 1);
        abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(&tmem_base_sh, 512);
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
            prefetch_tmap(&mQt); prefetch_tmap(&mKt); prefetch_tmap(&mQs); prefetch_tmap(&mKs);
            mbar_expect_tx(&bar_q, C::QT_BYTES + C::QS_BYTES);
#pragma unroll
            for (int b = 0; b < DT / 64; ++b) tma_load_3d(sQt + b * C::QBLK, &mQt, &bar_q, b * 64, q0, bh);
#pragma unroll
            for (int b = 0; b < DS / 64; ++b) tma_load_3d(sQs + b * C::QBLK, &mQs, &bar_q, b * 64, q0, bh);
            int issued = 0;
            for (int kt = 0; kt < n_kt; ++kt) {
                const int s = kt % C::NSTAGE, n = kt / C::NSTAGE;
                if (n > 0 && !mbar_wait(&bar_kempty[s], (n - 1) & 1, p.st, abort_v, 21)) break;
                uint8_t *st = sK + s * C::STAGE_BYTES;
                mbar_expect_tx(&bar_kfull[s], C::STAGE_BYTES);
#pragma unroll
                for (int b = 0; b < DT / 64; ++b)
                    tma_load_3d(st + b * C::KBLK, &mKt, &bar_kfull[s], b * 64, kt * C::BN, bh);
#pragma unroll
                for (int b = 0; b < DS / 64; ++b)
                    tma_load_3d(st + C::KT_BYTES + b * C::KBLK, &mKs, &bar_kfull[s], b * 64, kt * C::BN, bh);
                issued = kt + 1;
            }
            if (*abort_v) {
                DevStatus quick = p.st;
                quick.budget_ns = 50000000ull;
                volatile int never = 0;
                mbar_wait(&bar_q, 0, quick, &never, 21);
                for (int kt = (issued > C::NSTAGE ? issued - C::NSTAGE : 0); kt < issued; ++kt)
                    mbar_wait(&bar_kfull[kt % C::NSTAGE], (kt / C::NSTAGE) & 1, quick, &never, 21);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (elect_one()) {
            const uint32_t aQt = smem_u32(sQt), aQs = smem_u32(sQs);
            const uint32_t aDss = smem_u32(sDss), aDst = smem_u32(sDst);
            auto issue_s = [&](int kt) -> bool {
                const int s = kt % C::NSTAGE, n = kt / C::NSTAGE, buf = kt & 1, use = kt >> 1;
                if (!mbar_wait(&bar_kfull[s], n & 1, p.st, abort_v, 22)) return false;
                if (use > 0 && !mbar_wait(&bar_sempty[buf], (use - 1) & 1, p.st, abort_v, 23)) return false;
                tc_fence_after();
                const uint32_t aKt = smem_u32(sK + s * C::STAGE_BYTES), aKs = aKt + C::KT_BYTES;
#pragma unroll
                for (int kk = 0; kk < DT / 16; ++kk)
                    mma_bf16_ss(tmem + buf * 128, sw128_desc(aQt + (kk >> 2) * C::QBLK + (kk & 3) * 32, 16, 1024),
                                sw128_desc(aKt + (kk >> 2) * C::KBLK + (kk & 3) * 32, 16, 1024), C::IDESC_S, kk > 0);
#pragma unroll
                for (int kk = 0; kk < DS / 16; ++kk)
                    mma_bf16_ss(tmem + buf * 128 + 64,
                                sw128_desc(aQs + (kk >> 2) * C::QBLK + (kk & 3) * 32, 16, 1024),
                                sw128_desc(aKs + (kk >> 2) * C::KBLK + (kk & 3) * 32, 16, 1024), C::IDESC_S, kk > 0);
                mma_commit(&bar_sfull[buf]);
                return true;
            };
            bool ok = mbar_wait(&bar_q, 0, p.st, abort_v, 24);
            if (ok) ok = issue_s(0);
            for (int kt = 0; ok && kt < n_kt; ++kt) {
                if (kt + 1 < n_kt && !issue_s(kt + 1)) break;
                if (!mbar_wait(&bar_dsfull, kt & 1, p.st, abort_v, 25)) break;
                tc_fence_after();
                const int s = kt % C::NSTAGE;
                const uint32_t aKt = smem_u32(sK + s * C::STAGE_BYTES), aKs = aKt + C::KT_BYTES;
#pragma unroll
                for (int ks = 0; ks < C::BN / 16; ++ks)
                    mma_bf16_ss(tmem + C::TMEM_DQS, sw128_desc(aDss + ks * 32, 16, 1024),
                                sw128_desc(aKs + ks * 2048, C::KBLK, 1024), C::IDESC_QS, (kt > 0 || ks > 0));
                if (TEACHER) {
#pragma unroll
                    for (int ks = 0; ks < C::BN / 16; ++ks)
                        mma_bf16_ss(tmem + C::TMEM_DQT, sw128_desc(aDst + ks * 32, 16, 1024),
                                    sw128_desc(aKt + ks * 2048, C::KBLK, 1024), C::IDESC_QT, (kt > 0 || ks > 0));
                }
                mma_commit(&bar_dsempty);
                mma_commit(&bar_kempty[s]);
            }
            mma_commit(&bar_done);
        }
    } else {
        // ------------------------------------------------------------ gradient warpgroups (thread = query)
        // Warpgroup wg handles key columns [32 wg, 32 wg + 32) of every tile and
        // drains its share of the dQ columns at the end.
        const int wg = (warp - 2) >> 2;
        const int sub = warp & 3;
        const int row = sub * 32 + lane;
        const int gq = q0 + row;
        const int c0 = wg * 32;
        const uint32_t lane_base = tmem + ((uint32_t)(sub * 32) << 16);
        float Lt = 0.f, Ls = 0.f, g = 0.f, KL2 = 0.f;
        if (gq < p.N_Q) {
            const size_t r = (size_t)bh * p.N_Q + gq;
            Lt = p.lse_t[r] * kLog2eF;
            Ls = p.lse_s[r] * kLog2eF;
            g = p.dkl ? p.dkl[r] : p.g_const;
            KL2 = p.kl[r] * kLog2eF;
        }
        const int lim = p.causal ? min(p.N_K, gq + off + 1) : p.N_K;   // first hidden key
        bool ok = true;
        for (int kt = 0; kt < n_kt; ++kt) {
            const int buf = kt & 1, use = kt >> 1;
            if (!mbar_wait(&bar_sfull[buf], use & 1, p.st, abort_v, 26)) { ok = false; break; }
            tc_fence_after();
            const int kb = kt * C::BN + c0;
            const bool masked = (kb + 32 > p.N_K) || (p.causal && (kb + 31 > q0 + off));
            uint32_t ps[16], pt[16];
            {
                float ut[32], us[32];
                tmem_ld32(lane_base + buf * 128 + c0, ut);
                tmem_ld32(lane_base + buf * 128 + 64 + c0, us);
                tmem_ld_wait();
                if (masked) {
#pragma unroll
                    for (int k = 0; k < 32; k += 2) {
                        const int j = kb + k;
                        ds_pair<TEACHER, true>(ut[k], ut[k + 1], us[k], us[k + 1], p.ct, p.cs, Lt, Ls, g, KL2, j < lim,
                                               j + 1 < lim, ps[k >> 1], pt[k >> 1]);
                    }
                } else {
#pragma unroll
                    for (int k = 0; k < 32; k += 2)
                        ds_pair<TEACHER, false>(ut[k], ut[k + 1], us[k], us[k + 1], p.ct, p.cs, Lt, Ls, g, KL2, true,
                                                true, ps[k >> 1], pt[k >> 1]);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar_sempty[buf]);
            if (kt > 0 && !mbar_wait(&bar_dsempty, (kt - 1) & 1, p.st, abort_v, 27)) { ok = false; break; }
            store_row32(sDss, row, wg * 4, ps);
            if (TEACHER) store_row32(sDst, row, wg * 4, pt);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar_dsfull);
        }
        if (ok && mbar_wait(&bar_done, 0, p.st, abort_v, 28)) {
            tc_fence_after();
            const bool store = gq < p.N_Q;
            const size_t r = (size_t)bh * p.N_Q + (store ? gq : 0);
            constexpr int HS = DS / C::NWG, HT = DT / C::NWG;
            drain_row<HS>(lane_base + C::TMEM_DQS + wg * HS, p.out_s, p.dq_s + r * DS + wg * HS, store);
            if (TEACHER) drain_row<HT>(lane_base + C::TMEM_DQT + wg * HT, p.out_t, p.dq_t + r * DT + wg * HT, store);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace skl
