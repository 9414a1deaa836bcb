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
//       tiles: S^T = K Q^T (teacher and student), dS^T, dK += dS^T Q.
//       Thread = key row, so the per-query values (KL, the two log-sum-exps,
//       and g when it varies per row) come from a small per-stage table in
//       shared memory, read with one 16-byte broadcast load per four queries.
//       The persistent form (K in tensor memory), whose gradient warps are its
//       limit, instead adds the log-sum-exps to the logits with one extra
//       rank-1 MMA per tensor and tile: A = a constant [128 x 16] matrix whose
//       rows are (1, 1, 1, 0, ...), B = the tile's rows (h, m, l, 0, ...) with
//       h + m + l = -LSE / scale split into three bf16 terms (about fp32
//       precision), so the accumulator holds q.k - LSE / scale directly.
//   streamkl_bwd_dq_kernel   CTA = 128 queries of one head; loops over 64-key
//       tiles: S = Q K^T, dS, dQ += dS K.  Thread = query row; per-row
//       constants live in registers.
// Both recompute S: that costs one extra pair of QK^T products per element
// but removes the fp32 read-modify-write traffic a single kernel would need
// for the side it does not own (measured at ~5.8 TB/s of L2 reductions on
// B200, that traffic would cost more than the recompute).
//
// Pipeline (both kernels).  Tile t goes to TMEM buffer t & 1 (S_t in columns
// [0,64), S_s in [64,128) of the buffer); all four gradient warpgroups work on
// every tile, each on its own 16-column chunk, so sixteen warps share the
// exponentials of a tile while the MMA warp computes the logits of the next
// tile in the other buffer.  A warpgroup reads its chunk in 8-column pieces
// and writes the chunk's bf16 dS_s and dS_t (8 packed columns each) over its
// teacher logits, which only it reads; the MMA warp then uses those columns
// directly as the A operand of the gradient MMA (tcgen05.mma with A in tensor
// memory), so dS never touches shared memory.  The student half of the buffer
// is free as soon as every warp has read it, so the student logits of tile
// t+2 are issued then, during the dS math of tile t; because MMAs issued by
// one thread execute in order, the teacher logits of t+2 follow right after
// the gradient MMA of t, which leaves only half of the next logits on the
// critical path.  The two hand-offs of a tile ("student logits read", "dS
// written") go through named barriers where the resident operand is in
// shared memory (the d = 128 teacher-and-student forms), and through
// mbarriers polled by the MMA thread where it is in tensor memory.
#pragma once

#include <cuda_bf16.h>

#include "sm100.cuh"

namespace skl {

struct BwdParams {
    int BH, N_Q, N_K, causal, n_tiles;
    int H, Hkt, Hks;              // query heads per batch element, key heads of K_t and K_s
    const int *kv_len;            // per-batch key lengths (padding), or null
    int splits;                   // query-owner kernel: key ranges per query tile (1 = whole row)
    float ct, cs;                 // scale * log2(e)
    float out_t, out_s;           // output scales: scale_t * ln2 (teacher), scale_s (student)
    const float *kl, *lse_t, *lse_s, *dkl;
    float g_const;                // g when dkl == nullptr (times *g_dev when g_dev != nullptr)
    const float *g_dev;           // optional device scalar factor of g_const
    float inv_scale_t, inv_scale_s;
    float *dq_s, *dq_t, *dk_s, *dk_t;
    float *part_s, *part_t;       // splits > 1: per-split dQ partials [splits][BH*N_Q][d]
    const void *qt_raw, *kt_raw, *qs_raw, *ks_raw;   // the inputs as plain pointers (rows copied to TMEM)
    DevStatus st;
};

// The upstream gradient shared by all rows when no per-row dkl is given.
__device__ __forceinline__ float uniform_g(const BwdParams &p) {
    return p.g_dev ? p.g_const * __ldg(p.g_dev) : p.g_const;
}

constexpr float kLog2eF = 1.4426950408889634074f;

// x as three bf16 values h + m + l (each the rounding of what is left), packed
// as K elements 0..2 of a bf16 row (lower half first); the sum reproduces x to
// about 2^-24 relative, so a rank-1 MMA can add an fp32-accurate per-column
// offset to an accumulator.
__device__ __forceinline__ uint2 split3_bf16(float x) {
    const __nv_bfloat16 h = __float2bfloat16_rn(x);
    const float r1 = x - __bfloat162float(h);
    const __nv_bfloat16 m = __float2bfloat16_rn(r1);
    const __nv_bfloat16 l = __float2bfloat16_rn(r1 - __bfloat162float(m));
    return make_uint2((uint32_t)__bfloat16_as_ushort(h) | ((uint32_t)__bfloat16_as_ushort(m) << 16),
                      (uint32_t)__bfloat16_as_ushort(l));
}

// dS for two adjacent elements, packed as bf16x2 (lower half = first element).
// Per-element constants: L (log2-domain LSEs), g and KL*log2(e).
// With SCALE_G false the factor g is left out (dS / g is stored): the caller
// applies g to the accumulated gradient instead, which is exact whenever g is
// the same for every element the accumulator sums (a uniform g, or the
// per-row g of the query-owner kernel) and saves two multiplies per element.
template <bool TEACHER, bool MASKED, bool SCALE_G = true>
__device__ __forceinline__ void ds_pair(float ut0, float ut1, float us0, float us1, float ct, float cs, float Lt0,
                                        float Lt1, float Ls0, float Ls1, float g0, float g1, float K0, float K1,
                                        bool vis0, bool vis1, uint32_t &ps, uint32_t &pt) {
    const float at0 = fmaf(ut0, ct, -Lt0), at1 = fmaf(ut1, ct, -Lt1);
    const float as0 = fmaf(us0, cs, -Ls0), as1 = fmaf(us1, cs, -Ls1);
    float P0 = ex2(at0), P1 = ex2(at1);
    float Q0 = ex2(as0), Q1 = ex2(as1);
    if (MASKED) {
        P0 = vis0 ? P0 : 0.f; Q0 = vis0 ? Q0 : 0.f;
        P1 = vis1 ? P1 : 0.f; Q1 = vis1 ? Q1 : 0.f;
    }
    if (SCALE_G) {
        ps = pack_bf16(g0 * (Q0 - P0), g1 * (Q1 - P1));
        if (TEACHER) pt = pack_bf16((g0 * P0) * ((at0 - as0) - K0), (g1 * P1) * ((at1 - as1) - K1));
    } else {
        ps = pack_bf16(Q0 - P0, Q1 - P1);
        if (TEACHER) pt = pack_bf16(P0 * ((at0 - as0) - K0), P1 * ((at1 - as1) - K1));
    }
}

// ds_pair without g (SCALE_G false) on packed fp32 pairs: the same operations
// in the same order, so the same results, with the element-wise arithmetic
// issued as f32x2 instructions.  ct2, cs2: splatted scales; nLt2, nLs2: minus
// the log2-domain LSEs of the two elements (zero where a bias MMA already
// subtracted them); K2: KL log2(e) of the two elements' rows.
template <bool TEACHER, bool MASKED>
__device__ __forceinline__ void ds_pair_x2(float ut0, float ut1, float us0, float us1, uint64_t ct2, uint64_t cs2,
                                           uint64_t nLt2, uint64_t nLs2, uint64_t K2, bool vis0, bool vis1,
                                           uint32_t &ps, uint32_t &pt) {
    const uint64_t at = f2fma(f2pack(ut0, ut1), ct2, nLt2);
    const uint64_t as = f2fma(f2pack(us0, us1), cs2, nLs2);
    const float2 a = f2unpack(at), b = f2unpack(as);
    float P0 = ex2(a.x), P1 = ex2(a.y);
    float Q0 = ex2(b.x), Q1 = ex2(b.y);
    if (MASKED) {
        P0 = vis0 ? P0 : 0.f; Q0 = vis0 ? Q0 : 0.f;
        P1 = vis1 ? P1 : 0.f; Q1 = vis1 ? Q1 : 0.f;
    }
    const uint64_t P = f2pack(P0, P1), Q = f2pack(Q0, Q1);
    const float2 d = f2unpack(f2sub(Q, P));
    ps = pack_bf16(d.x, d.y);
    if (TEACHER) {
        const float2 e = f2unpack(f2mul(P, f2sub(f2sub(at, as), K2)));
        pt = pack_bf16(e.x, e.y);
    }
}

// The two chunk routines below turn one CWID-column chunk of a warpgroup's S
// columns (teacher logits at `at`, student at `as`) into this thread's CWID dS
// values.  The logits are read in pieces of PW columns and each piece's load
// is issued before the previous piece is computed, so the tensor-memory
// latency overlaps the arithmetic.  As soon as the last piece has landed the
// warp signals `rel` (an mbarrier, or a named barrier: its student logits are
// no longer needed, so the next tile's student logits may overwrite them);
// once the whole chunk is
// computed, the packed bf16 dS_s (CWID/2 columns) and dS_t (the next CWID/2)
// are stored over this chunk's teacher logits, which only this warpgroup
// reads.
constexpr int kBwdPiece = 8;

__device__ __forceinline__ void release_student_logits(uint64_t *sfree) {
    tc_fence_before();
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(sfree);
}

// The same on named barrier `id` (every lane arrives; -1: nobody waits for
// this tile's release, so no arrival), with n threads taking part.
struct NamedRel { int id; };
__device__ __forceinline__ void release_student_logits(NamedRel r, int n) {
    if (r.id >= 0) {
        tc_fence_before();
        named_arrive(r.id, n);
    }
}
__device__ __forceinline__ void release_student_logits(uint64_t *sfree, int) { release_student_logits(sfree); }

template <bool TEACHER, int CWID>
__device__ __forceinline__ void store_ds(uint32_t at, const uint32_t (&ps)[CWID / 2], const uint32_t (&pt)[CWID / 2]) {
    static_assert(CWID == 16 || CWID == 32, "8 or 16 packed columns");
    if constexpr (CWID == 16) {
        tmem_st8(at, ps);
        if (TEACHER) tmem_st8(at + 8, pt);
    } else {
        tmem_st16(at, ps);
        if (TEACHER) tmem_st16(at + 16, pt);
    }
}

// Query-owner chunk (thread = query row; constants per row, keys kb ..
// kb+CWID-1, keys >= lim hidden).  The row's g multiplies its dQ at the end.
template <bool TEACHER, bool MASKED, int CWID, int PW = kBwdPiece, typename Rel>
__device__ __forceinline__ void dq_chunk(uint32_t at, uint32_t as, float ct, float cs, float Lt, float Ls, float g,
                                         float KL2, int kb, int lim, Rel rel, int nsync) {
    constexpr int NP = CWID / PW;
    float ut[2][PW], us[2][PW];
    uint32_t ps[CWID / 2], pt[CWID / 2];
    tmem_ld<PW>(at, ut[0]);
    tmem_ld<PW>(as, us[0]);
    tmem_ld_wait_bind(ut[0], us[0]);
    if (NP == 1) release_student_logits(rel, nsync);
#pragma unroll
    for (int pc = 0; pc < NP; ++pc) {
        const int cur = pc & 1;
        if (pc + 1 < NP) {
            tmem_ld<PW>(at + PW * (pc + 1), ut[cur ^ 1]);
            tmem_ld<PW>(as + PW * (pc + 1), us[cur ^ 1]);
        }
#pragma unroll
        for (int k = 0; k < PW; k += 2) {
            const int j = kb + PW * pc + k, o = (PW * pc + k) >> 1;
            ds_pair_x2<TEACHER, MASKED>(ut[cur][k], ut[cur][k + 1], us[cur][k], us[cur][k + 1], f2splat(ct),
                                        f2splat(cs), f2splat(-Lt), f2splat(-Ls), f2splat(KL2), j < lim, j + 1 < lim,
                                        ps[o], pt[o]);
        }
        if (pc + 1 < NP) {
            tmem_ld_wait_bind(ut[cur ^ 1], us[cur ^ 1]);
            if (pc + 2 == NP) release_student_logits(rel, nsync);
        }
    }
    store_ds<TEACHER, CWID>(at, ps, pt);
}

// Key-owner chunk (thread = key row).  The per-query values come from
// shared-memory tables: KL log2(e) (`ktab`), g when it varies per row (G_ROW:
// `gtab`; otherwise g is uniform and the caller applies it to the accumulated
// dK instead) and, with LTAB, -LSE_t log2(e) and -LSE_s log2(e) (`ltab`,
// `stab`), folded into the first fused multiply-add; without LTAB the logits
// already carry -LSE / scale (a rank-1 bias MMA added it).
// Every thread of the warp reads the same four floats with one 16-byte
// broadcast load per four columns (a quarter of the load instructions of
// 4-byte loads, for the same shared-memory wavefronts per value; measured
// 2 % faster).  Columns q < qmin, relative to the chunk, are hidden.
template <bool TEACHER, bool MASKED, bool G_ROW, int CWID, int PW = kBwdPiece, typename Rel, bool LTAB = false>
__device__ __forceinline__ void dkv_chunk(uint32_t at, uint32_t as, float ct, float cs, const float *ktab,
                                          const float *gtab, float g_uni, int qmin, Rel rel, int nsync,
                                          const float *ltab = nullptr, const float *stab = nullptr) {
    constexpr int NP = CWID / PW;
    float ut[2][PW], us[2][PW];
    float4 k4 = make_float4(0.f, 0.f, 0.f, 0.f);   // KL log2(e) of four query columns
    float4 l4 = make_float4(0.f, 0.f, 0.f, 0.f);   // LTAB: -LSE_t log2(e) of the same four columns
    float4 s4 = make_float4(0.f, 0.f, 0.f, 0.f);   // LTAB: -LSE_s log2(e)
    uint32_t ps[CWID / 2], pt[CWID / 2];
    tmem_ld<PW>(at, ut[0]);
    tmem_ld<PW>(as, us[0]);
    tmem_ld_wait_bind(ut[0], us[0]);
    if (NP == 1) release_student_logits(rel, nsync);
#pragma unroll
    for (int pc = 0; pc < NP; ++pc) {
        const int cur = pc & 1;
        if (pc + 1 < NP) {
            tmem_ld<PW>(at + PW * (pc + 1), ut[cur ^ 1]);
            tmem_ld<PW>(as + PW * (pc + 1), us[cur ^ 1]);
        }
#pragma unroll
        for (int k = 0; k < PW; k += 2) {
            const int q = PW * pc + k;
            float2 K = make_float2(0.f, 0.f), NL = make_float2(0.f, 0.f), NS = make_float2(0.f, 0.f);
            if constexpr (TEACHER) {
                if ((q & 3) == 0) {
                    k4 = ld_shared_v4(ktab + q);
                    K = make_float2(k4.x, k4.y);
                } else {
                    K = make_float2(k4.z, k4.w);
                }
            }
            if constexpr (LTAB) {
                if ((q & 3) == 0) {
                    l4 = ld_shared_v4(ltab + q);
                    s4 = ld_shared_v4(stab + q);
                    NL = make_float2(l4.x, l4.y);
                    NS = make_float2(s4.x, s4.y);
                } else {
                    NL = make_float2(l4.z, l4.w);
                    NS = make_float2(s4.z, s4.w);
                }
            }
            const float2 G = G_ROW ? *reinterpret_cast<const float2 *>(gtab + q) : make_float2(g_uni, g_uni);
            if constexpr (G_ROW)
                ds_pair<TEACHER, MASKED, true>(ut[cur][k], ut[cur][k + 1], us[cur][k], us[cur][k + 1], ct, cs,
                                               LTAB ? -NL.x : 0.f, LTAB ? -NL.y : 0.f, LTAB ? -NS.x : 0.f,
                                               LTAB ? -NS.y : 0.f, G.x, G.y, K.x, K.y, q >= qmin, q + 1 >= qmin,
                                               ps[q >> 1], pt[q >> 1]);
            else
                ds_pair_x2<TEACHER, MASKED>(ut[cur][k], ut[cur][k + 1], us[cur][k], us[cur][k + 1], f2splat(ct),
                                            f2splat(cs), LTAB ? f2pack(NL.x, NL.y) : 0ull,
                                            LTAB ? f2pack(NS.x, NS.y) : 0ull, f2pack(K.x, K.y), q >= qmin,
                                            q + 1 >= qmin, ps[q >> 1], pt[q >> 1]);
        }
        if (pc + 1 < NP) {
            tmem_ld_wait_bind(ut[cur ^ 1], us[cur ^ 1]);
            if (pc + 2 == NP) release_student_logits(rel, nsync);
        }
    }
    store_ds<TEACHER, CWID>(at, ps, pt);
}

// Warpgroup layout of both backward kernels: tiles alternate between two TMEM
// logit buffers; kBwdParities groups of warpgroups take turns on the tiles
// (1: every warpgroup works on every tile) and the kBwdHalves warpgroups of a
// group split a tile's 64 columns into chunks of 64 / kBwdHalves.
constexpr int kBwdParities = 1;
constexpr int kBwdHalves = 4;
constexpr int kBwdChunk = 64 / kBwdHalves;

// Writes NCOLS (16 or 32) accumulator columns of this warp's 32 TMEM lanes
// (rows row0 .. row0+31 of the output, of which the first nvalid exist) to
// global memory, scaled by `scale` (per thread = per row), or zeros for the
// rows whose thread passes `zero` (a padding key, or no visible pair at all:
// the accumulator is then not read as a value, so nothing in it can leak).  Each thread first
// puts its row into a per-warp staging tile in shared memory with 16-byte
// stores (row stride NCOLS + 4 floats: rows stay 16-byte aligned and the eight
// rows written by a quarter-warp fall into different banks), then the warp
// stores the tile with 16-byte loads and stores, 32 / (NCOLS / 4) whole row
// segments per instruction, so every global store covers complete 64- or
// 128-byte runs.  `dst` points at column 0 of row row0 and is 16-byte
// aligned, as is `ld` * 4 bytes, the row stride.  `lim` is one past the end
// of the output tensor (checked in the bounds-checked build).
constexpr int kDrainPad = 4;

// Named barriers of the backward kernels' per-tile hand-off: "dS written" of
// tile t on id nb_dsfull(t) and "student logits read" on nb_ssfree(t), four
// ids of each kind used in turn.  The 16 gradient warps arrive (bar.arrive),
// the whole MMA warp waits (bar.sync): kNbCount threads.  A gradient warp's
// arrivals run at most two tiles ahead of the MMA warp's waits (tile t's
// logits are committed only after the MMA warp has passed tile t-2), so
// while their logits come, no id is reused before its phase has completed.
// A warp whose bounded wait gave up no longer waits for logits; it takes part
// in each remaining tile's barriers with bar.sync, which cannot complete
// before the MMA warp's wait on the same tile, so from its first such tile on
// it stays in step.  With one id per logit buffer that first tile (t+2 after
// its last arrival for t) would share the id of a phase still open: the
// phase would complete with the arrivals of two tiles and the MMA warp's
// later wait never (tests/test_handoff_protocol.py runs the protocol as a
// model).  Measured against mbarriers polled by the MMA thread (a per-tile
// timeline of the query-owner kernel at 8k, d = 128, teacher and student):
// the MMA thread passed an already completed mbarrier ~240 clk after the last
// arrival, a named barrier ~35 clk after it.
constexpr int kNbDsfullBase = 1, kNbSsfreeBase = 5, kNbCount = 32 * (16 + 1);
__host__ __device__ constexpr int nb_dsfull(int t) { return kNbDsfullBase + (t & 3); }
__host__ __device__ constexpr int nb_ssfree(int t) { return kNbSsfreeBase + (t & 3); }


template <int NCOLS>
__device__ __forceinline__ void drain_rows(uint32_t taddr, float scale, float *dst, size_t ld, int nvalid,
                                           float *stage, int lane, bool zero, const float *lim, uint32_t *word) {
    static_assert(NCOLS == 16 || NCOLS == 32, "16 or 32 columns");
    constexpr int SP = NCOLS + kDrainPad, V = NCOLS / 4, RPI = 32 / V;
    float4 *mine = reinterpret_cast<float4 *>(stage + lane * SP);
#pragma unroll
    for (int c = 0; c < NCOLS; c += 16) {
        float v[16];
        tmem_ld16(taddr + c, v);
        tmem_ld_wait();
#pragma unroll
        for (int k = 0; k < 4; ++k)
            mine[c / 4 + k] = zero ? make_float4(0.f, 0.f, 0.f, 0.f)
                                   : make_float4(v[4 * k] * scale, v[4 * k + 1] * scale, v[4 * k + 2] * scale,
                                                 v[4 * k + 3] * scale);
    }
    __syncwarp();
    const int rr = lane / V, c4 = (lane % V) * 4;
#pragma unroll
    for (int j = 0; j < 32 / RPI; ++j) {
        const int r = j * RPI + rr;
        if (r < nvalid && bound_ok(dst + (size_t)r * ld + c4 + 4 <= lim, word, kSiteDrain))
            *reinterpret_cast<float4 *>(dst + (size_t)r * ld + c4) =
                *reinterpret_cast<const float4 *>(stage + r * SP + c4);
    }
    __syncwarp();
}

// Writes NCOLS (16 or 32) accumulator columns of this thread's TMEM lane,
// scaled by `scale` (or zeros when `zero`), to its output row at `dst` (when
// `valid`), straight from registers: 32-byte stores when `dst` is 32-byte aligned (whole sectors),
// else 16-byte stores.
template <int NCOLS>
__device__ __forceinline__ void drain_row(uint32_t taddr, float scale, float *dst, bool valid, bool zero,
                                          const float *lim, uint32_t *word) {
    static_assert(NCOLS == 16 || NCOLS == 32, "16 or 32 columns");
    const bool a32 = (reinterpret_cast<uintptr_t>(dst) & 31) == 0;
#pragma unroll
    for (int c = 0; c < NCOLS; c += 16) {
        float v[16];
        tmem_ld16(taddr + c, v);
        tmem_ld_wait();
#pragma unroll
        for (int k = 0; k < 16; ++k) v[k] = zero ? 0.f : v[k] * scale;
        if (valid && bound_ok(dst + c + 16 <= lim, word, kSiteDrain)) {
            if (a32) {
                st_global_v8(dst + c, v[0], v[1], v[2], v[3], v[4], v[5], v[6], v[7]);
                st_global_v8(dst + c + 8, v[8], v[9], v[10], v[11], v[12], v[13], v[14], v[15]);
            } else {
#pragma unroll
                for (int k = 0; k < 16; k += 4)
                    *reinterpret_cast<float4 *>(dst + c + k) = make_float4(v[k], v[k + 1], v[k + 2], v[k + 3]);
            }
        }
    }
}

// TMEM column (within a buffer) of the packed bf16 dS_s for keys/queries
// [16 ks, 16 ks + 16): each warpgroup's 16-column chunk of the teacher logits
// holds its 8 packed dS_s columns, then its 8 packed dS_t columns.
static_assert(kBwdChunk == 16, "dS layout assumes 16-column chunks");
__host__ __device__ constexpr uint32_t ds_col_s(int ks) { return (uint32_t)(16 * ks); }
__host__ __device__ constexpr uint32_t ds_col_t(int ks) { return (uint32_t)(16 * ks + 8); }

// ============================================================================ dK kernel
template <int DT, int DS, bool TEACHER>
struct DkvCfg {
    static constexpr int BN = 128, BM = 64;       // keys per CTA, queries per tile
    static constexpr int KBLK = 128 * 128;         // [128 rows][64] bf16 box
    static constexpr int QBLK = 64 * 128;          // [64 rows][64] bf16 box
    // Tensor memory: logit buffers [0, 256), dK_s, dK_t, and, when they fit
    // (K_TMEM: the student-only and d = 64 cases), this CTA's K_t and K_s rows
    // as packed bf16, so the logit MMAs read only the Q tile from shared memory.
    static constexpr uint32_t TMEM_DKS = 256, TMEM_DKT = 256 + DS;
    static constexpr uint32_t TMEM_KT = TMEM_DKT + (TEACHER ? DT : 0), TMEM_KS = TMEM_KT + DT / 2;
    static constexpr bool K_TMEM = TMEM_KS + DS / 2 <= 512;
    static constexpr int KT_BYTES = K_TMEM ? 0 : BN * DT * 2, KS_BYTES = K_TMEM ? 0 : BN * DS * 2;
    static constexpr int QT_BYTES = BM * DT * 2, QS_BYTES = BM * DS * 2;
    static constexpr int STAGE_TMA = QT_BYTES + QS_BYTES;
    // The per-query log-sum-exps reach the logits in one of two ways.
    // LSE_TAB (the one-item kernel, K in shared memory): from a per-stage table
    // that the gradient warps read with the KL values (16-byte broadcast
    // loads), subtracted in their first fused multiply-add.  Otherwise (the
    // persistent kernel): by one rank-1 bias MMA per tensor and tile.  The
    // one-item kernel at d = 128 is limited by its MMAs, the persistent one by
    // its gradient warps, so each takes the work where it has room.
    static constexpr bool LSE_TAB = !K_TMEM;
    static constexpr int BIAS_BYTES = LSE_TAB ? 0 : BM * 16 * 2;  // [64 queries][16] bf16, unswizzled K-major
    // per query: KL log2(e), then g, then (LSE_TAB) -LSE_t log2(e) and -LSE_s log2(e)
    static constexpr int GK_BYTES = BM * (LSE_TAB ? 16 : 8);
    static constexpr int BIAS_T = STAGE_TMA, BIAS_S = BIAS_T + BIAS_BYTES, GK = BIAS_S + BIAS_BYTES;
    static constexpr int STAGE_BYTES = ((GK + GK_BYTES + 1023) / 1024) * 1024;
    static constexpr int ONES_BYTES = LSE_TAB ? 0 : BN * 16 * 2;  // [128 keys][16] bf16 rows (1, 1, 1, 0, ...)
    // K_STAGED (persistent form, K in tensor memory): the next item's K rows
    // land in a staging area by TMA (K_t boxes, then K_s boxes) and the
    // gradient warps copy them into tensor memory.  Used when the Q ring keeps
    // at least five stages beside the area; otherwise the gradient warps read
    // the rows from global memory (fewer stages cost more than the copy saves).
    static constexpr int KST_FULL = K_TMEM ? BN * (DT + DS) * 2 : 0;
    static constexpr bool K_STAGED =
        K_TMEM && (224 * 1024 - (KT_BYTES + KS_BYTES + ONES_BYTES + KST_FULL)) / STAGE_BYTES >= 5;
    static constexpr int KST_BYTES = K_STAGED ? KST_FULL : 0;
    static constexpr int FIXED = KT_BYTES + KS_BYTES + ONES_BYTES + KST_BYTES;
    static constexpr int NS_RAW = (224 * 1024 - FIXED) / STAGE_BYTES;
    static constexpr int NSTAGE = NS_RAW < 2 ? 2 : (NS_RAW > 6 ? 6 : NS_RAW);
    // the student logits of tile t+2 are issued before the gradient MMA of
    // tile t releases its stage, so t+2 must not need that stage
    static_assert(NSTAGE >= 3, "stage ring too shallow for the early student logits");
    static_assert(NSTAGE * STAGE_BYTES >= 16 * 32 * (32 + kDrainPad) * 4, "stage ring doubles as the drain staging area");
    static constexpr int SMEM = FIXED + NSTAGE * STAGE_BYTES + 1024;
    static constexpr int NH = kBwdHalves, NWG = kBwdParities * kBwdHalves, CW = BM / NH;
    static constexpr int THREADS = 64 + 128 * NWG;
    static constexpr uint32_t IDESC_S = idesc_bf16(128, BM, 0, 0);
    static constexpr uint32_t IDESC_KS = idesc_bf16(128, DS, 0, 1);
    static constexpr uint32_t IDESC_KT = idesc_bf16(128, DT, 0, 1);
};

// PAD: the problem has per-batch key lengths (padding).  A separate
// instantiation, because the padding checks cost registers that the tile loop
// of the d = 128 teacher-and-student form, at the register limit, does not have.
template <int DT, int DS, bool TEACHER, bool PAD>
__global__ void __launch_bounds__(DkvCfg<DT, DS, TEACHER>::THREADS, 1)
    streamkl_bwd_dkv_kernel(const __grid_constant__ CUtensorMap mQt, const __grid_constant__ CUtensorMap mKt,
                            const __grid_constant__ CUtensorMap mQs, const __grid_constant__ CUtensorMap mKs,
                            const BwdParams p) {
    using C = DkvCfg<DT, DS, TEACHER>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sKt = smem;
    uint8_t *sKs = sKt + C::KT_BYTES;
    uint8_t *sQ = sKs + C::KS_BYTES;               // stages: Q_t, Q_s, then per query {KL, g, -LSE_t, -LSE_s}

    // The per-tile hand-off between the gradient warps and the MMA warp ("dS
    // written", "student logits read") goes through named barriers
    // nb_dsfull(t) and nb_ssfree(t).
    __shared__ uint64_t bar_k, bar_qfull[C::NSTAGE], bar_qempty[C::NSTAGE], bar_sfull[2];
    __shared__ uint64_t bar_done;
    __shared__ uint64_t bar_quiet;                 // the MMA thread's issued MMAs have completed
    __shared__ uint32_t tmem_base_sh;
    __shared__ int abort_flag;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // tensors behind the four maps (bounds-checked build)
    const MapDims mdQt{DT, p.N_Q, p.BH}, mdQs{DS, p.N_Q, p.BH};
    const MapDims mdKt{DT, p.N_K, p.BH / p.H * p.Hkt}, mdKs{DS, p.N_K, p.BH / p.H * p.Hks};
    const int kt_idx = (int)(blockIdx.x / p.BH);   // low key tiles see the most queries: run them first
    const int bh = (int)(blockIdx.x % p.BH);
    const int k0 = kt_idx * C::BN;
    const int off = p.N_K - p.N_Q;
    const int n_qt_all = (p.N_Q + C::BM - 1) / C::BM;
    const int first_qt = p.causal ? max(0, k0 - off) / C::BM : 0;
    const int n_qt = max(0, n_qt_all - first_qt);
    const int bkt = key_head(bh, p.H, p.Hkt), bks = key_head(bh, p.H, p.Hks);   // this head's key heads
    if constexpr (PAD) {
        // A CTA whose keys are all padding has no visible pair: it writes its
        // zero dK rows and returns before any set-up (a whole-CTA decision, so
        // no barrier, copy or tensor memory is involved yet).
        const int nk = key_count(p.kv_len, bh / p.H, p.N_K, p.st.word, threadIdx.x == 0 && kt_idx == 0);
        if (k0 >= nk) {
            const int rows = min(C::BN, p.N_K - k0);
            if (!bound_ok(bh < p.BH && k0 >= 0 && rows > 0, p.st.word, kSiteZero)) return;
            float4 *ds4 = reinterpret_cast<float4 *>(p.dk_s + ((size_t)bh * p.N_K + k0) * DS);
            for (int e = threadIdx.x; e < rows * DS / 4; e += C::THREADS) ds4[e] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (TEACHER) {
                float4 *dt4 = reinterpret_cast<float4 *>(p.dk_t + ((size_t)bh * p.N_K + k0) * DT);
                for (int e = threadIdx.x; e < rows * DT / 4; e += C::THREADS) dt4[e] = make_float4(0.f, 0.f, 0.f, 0.f);
            }
            return;
        }
    }

    // Set-up.  Each warp has its own part, and the block barrier below waits
    // for the slowest: issuing a TMA copy takes a while, so before the barrier
    // only the copies the first logits need are issued (the resident K tile
    // and the first Q stage); the producer issues the rest after it.
    if (warp == 0) {
        if (lane == 0) {
            mbar_init(&bar_k, 1);
            for (int s = 0; s < C::NSTAGE; ++s) {
                mbar_init(&bar_qfull[s], 1 + 32);      // TMA expect_tx + every producer lane (constants)
                mbar_init(&bar_qempty[s], 1);
            }
            for (int b = 0; b < 2; ++b) {
                mbar_init(&bar_sfull[b], 1);
            }
            mbar_init(&bar_done, 1);
            mbar_init(&bar_quiet, 1);
            abort_flag = 0;
            fence_barrier_init();
            if (!C::K_TMEM) {
                prefetch_tmap(&mKt); prefetch_tmap(&mKs);
                mbar_expect_tx(&bar_k, C::KT_BYTES + C::KS_BYTES);
#pragma unroll
                for (int b = 0; b < DT / 64; ++b) tma_load_3d(sKt + b * C::KBLK, &mKt, &bar_k, b * 64, k0, bkt, mdKt, p.st.word);
#pragma unroll
                for (int b = 0; b < DS / 64; ++b) tma_load_3d(sKs + b * C::KBLK, &mKs, &bar_k, b * 64, k0, bks, mdKs, p.st.word);
            }
            prefetch_tmap(&mQt); prefetch_tmap(&mQs);
            if (n_qt > 0) {
                mbar_expect_tx(&bar_qfull[0], C::STAGE_TMA);
#pragma unroll
                for (int b = 0; b < DT / 64; ++b)
                    tma_load_3d(sQ + b * C::QBLK, &mQt, &bar_qfull[0], b * 64, first_qt * C::BM, bh, mdQt, p.st.word);
#pragma unroll
                for (int b = 0; b < DS / 64; ++b)
                    tma_load_3d(sQ + C::QT_BYTES + b * C::QBLK, &mQs, &bar_qfull[0], b * 64, first_qt * C::BM, bh, mdQs, p.st.word);
            }
        }
    } else if (warp == 1) {
        tmem_alloc(&tmem_base_sh, 512);
        tmem_relinquish();
    }
    static_assert(C::LSE_TAB, "the one-item kernel reads the log-sum-exps from tables (no MMA operands to set up)");
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base_sh;
    volatile int *abort_v = &abort_flag;
    if constexpr (C::K_TMEM) {
        if (warp >= 2) {
            const int wg = (warp - 2) >> 2, sub = warp & 3;
            resident_to_tmem<DT>(tmem, C::TMEM_KT, p.kt_raw, bkt, p.N_K, k0, wg, sub, lane, mdKt.n2, p.st.word);
            resident_to_tmem<DS>(tmem, C::TMEM_KS, p.ks_raw, bks, p.N_K, k0, wg, sub, lane, mdKs.n2, p.st.word);
            tmem_st_wait();
        }
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    }

    if (warp == 0) {
        // ------------------------------------------------------------ producer (TMA + per-query constants)
        // Per-query constants of a tile: lane l handles queries l and l + 32.  They
        // are fetched from global memory two tiles ahead into registers, with loads
        // the compiler may not move (ld_now), so that their latency overlaps the
        // tiles in between instead of stalling the ring.
        const float g_all = uniform_g(p);
        auto load_consts = [&](int t, float4 (&v)[2]) {   // raw {lse_t, lse_s, g, kl}
            const int q0 = (first_qt + t) * C::BM;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int i = q0 + lane + 32 * h;
                v[h] = make_float4(0.f, 0.f, 0.f, 0.f);        // rows past N_Q: g = 0, so dS = 0
                if (t < n_qt && i < p.N_Q && bound_ok(bh < p.BH && i >= 0, p.st.word, kSiteConst)) {
                    const size_t r = (size_t)bh * p.N_Q + i;
                    v[h].x = ld_now(p.lse_t + r);
                    v[h].y = ld_now(p.lse_s + r);
                    v[h].z = p.dkl ? ld_now(p.dkl + r) : g_all;
                    v[h].w = ld_now(p.kl + r);
                }
            }
        };
        float4 c0[2], c1[2], c2[2];
        load_consts(0, c1);
        load_consts(1, c2);
        int issued = 0;
        for (int t = 0; t < n_qt; ++t) {
            const int s = t % C::NSTAGE, n = t / C::NSTAGE;
            const int q0 = (first_qt + t) * C::BM;
            c0[0] = c1[0]; c0[1] = c1[1];
            c1[0] = c2[0]; c1[1] = c2[1];
            load_consts(t + 2, c2);
            if (n > 0 && !mbar_wait(&bar_qempty[s], (n - 1) & 1, p.st, abort_v, 11)) break;
            uint8_t *st = sQ + s * C::STAGE_BYTES;
            if (lane == 0 && t > 0) {            // the first stage was issued during set-up
                mbar_expect_tx(&bar_qfull[s], C::STAGE_TMA);
#pragma unroll
                for (int b = 0; b < DT / 64; ++b)
                    tma_load_3d(st + b * C::QBLK, &mQt, &bar_qfull[s], b * 64, q0, bh, mdQt, p.st.word);
#pragma unroll
                for (int b = 0; b < DS / 64; ++b)
                    tma_load_3d(st + C::QT_BYTES + b * C::QBLK, &mQs, &bar_qfull[s], b * 64, q0, bh, mdQs, p.st.word);
            }
            float *ktab = reinterpret_cast<float *>(st + C::GK), *gtab = ktab + C::BM;
            float *ltab = gtab + C::BM, *stab = ltab + C::BM;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int q = lane + 32 * h;
                ktab[q] = c0[h].w * kLog2eF;
                gtab[q] = c0[h].z;
                ltab[q] = -c0[h].x * kLog2eF;
                stab[q] = -c0[h].y * kLog2eF;
            }
            mbar_arrive(&bar_qfull[s]);
            issued = t + 1;
        }
        if (*abort_v && lane == 0) {
            DevStatus quick = p.st;
            quick.budget_ns = 50000000ull;
            volatile int never = 0;
            if (!C::K_TMEM) mbar_wait(&bar_k, 0, quick, &never, 11);
            for (int t = (issued > C::NSTAGE ? issued - C::NSTAGE : 0); t < issued; ++t)
                mbar_wait(&bar_qfull[t % C::NSTAGE], (t / C::NSTAGE) & 1, quick, &never, 11);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        // Descriptors are built once (warp-uniform) and advanced by constant offsets.
        const uint64_t dKt = sw128_desc(smem_u32(sKt), 16, 1024), dKs = sw128_desc(smem_u32(sKs), 16, 1024);
        const uint64_t dQ0 = sw128_desc(smem_u32(sQ), 16, 1024);          // K-major view of a stage
        const uint64_t dQ0mn = sw128_desc(smem_u32(sQ), C::QBLK, 1024);   // MN-major view of a stage
        const bool leader = elect_one();
        const int leader_lane = __ffs(__ballot_sync(0xffffffffu, leader)) - 1;
        {
            // Student S^T of tile t (plus its rank-1 bias -LSE_s / scale_s) into
            // columns [64, 128) of buffer t & 1, once the tile's Q stage has landed.
            auto issue_ss = [&](int t) -> bool {
                const int s = t % C::NSTAGE, n = t / C::NSTAGE, buf = t & 1;
                if (!mbar_wait(&bar_qfull[s], n & 1, p.st, abort_v, 12)) return false;
                tc_fence_after();
                const uint64_t dQs = desc_add(dQ0, s * C::STAGE_BYTES + C::QT_BYTES);
#pragma unroll
                for (int kk = 0; kk < DS / 16; ++kk) {
                    const uint64_t b = desc_add(dQs, (kk >> 2) * C::QBLK + (kk & 3) * 32);
                    if constexpr (C::K_TMEM)
                        mma_bf16_ts(tmem + buf * 128 + 64, tmem + C::TMEM_KS + kk * 8, b, C::IDESC_S, kk > 0);
                    else
                        mma_bf16_ss(tmem + buf * 128 + 64, desc_add(dKs, (kk >> 2) * C::KBLK + (kk & 3) * 32), b,
                                    C::IDESC_S, kk > 0);
                }
                return true;
            };
            // Teacher S^T (plus bias) into columns [0, 64), then signal the tile.
            auto issue_st = [&](int t) {
                const int s = t % C::NSTAGE, buf = t & 1;
                const uint64_t dQt = desc_add(dQ0, s * C::STAGE_BYTES);
#pragma unroll
                for (int kk = 0; kk < DT / 16; ++kk) {
                    const uint64_t b = desc_add(dQt, (kk >> 2) * C::QBLK + (kk & 3) * 32);
                    if constexpr (C::K_TMEM)
                        mma_bf16_ts(tmem + buf * 128, tmem + C::TMEM_KT + kk * 8, b, C::IDESC_S, kk > 0);
                    else
                        mma_bf16_ss(tmem + buf * 128, desc_add(dKt, (kk >> 2) * C::KBLK + (kk & 3) * 32), b,
                                    C::IDESC_S, kk > 0);
                }
                mma_commit(&bar_sfull[buf]);
            };
            bool ok = true;
            if (leader) {
                ok = C::K_TMEM || mbar_wait(&bar_k, 0, p.st, abort_v, 14);
                for (int t = 0; ok && t < 2 && t < n_qt; ++t) {
                    ok = issue_ss(t);
                    if (ok) issue_st(t);
                }
            }
            ok = __shfl_sync(0xffffffffu, ok, leader_lane);
            // The whole warp takes part in the named barriers; after a failed
            // wait it keeps taking part (issuing nothing), so that the gradient
            // warps, which make the same arrivals in any case, never wait on it.
            for (int t = 0; t < n_qt; ++t) {
                const int buf = t & 1, s = t % C::NSTAGE;
                const bool next = t + 2 < n_qt;
                // The student logits of tile t+2 go into this buffer as soon as every
                // warp has read tile t's (they keep their dS in the teacher half).
                __syncwarp();
                if (next) named_sync(nb_ssfree(t), kNbCount);
                if (ok && next) {
                    tc_fence_after();
                    bool r = true;
                    if (leader) r = issue_ss(t + 2);
                    ok = __shfl_sync(0xffffffffu, r, leader_lane);
                }
                named_sync(nb_dsfull(t), kNbCount);
                if (ok && leader) {
                    tc_fence_after();
                    const uint64_t mQt = desc_add(dQ0mn, s * C::STAGE_BYTES), mQs = desc_add(mQt, C::QT_BYTES);
                    // dK_s += dS_s^T Q_s : A = dS_s^T from TMEM (buffer columns [0,32)), B = Q_s (MN-major)
#pragma unroll
                    for (int ks = 0; ks < C::BM / 16; ++ks)
                        mma_bf16_ts(tmem + C::TMEM_DKS, tmem + buf * 128 + ds_col_s(ks), desc_add(mQs, ks * 2048),
                                    C::IDESC_KS, (t > 0 || ks > 0));
                    if (TEACHER) {
#pragma unroll
                        for (int ks = 0; ks < C::BM / 16; ++ks)
                            mma_bf16_ts(tmem + C::TMEM_DKT, tmem + buf * 128 + ds_col_t(ks), desc_add(mQt, ks * 2048),
                                        C::IDESC_KT, (t > 0 || ks > 0));
                    }
                    mma_commit(&bar_qempty[s]);
                    if (next) issue_st(t + 2);
                }
                __syncwarp();
            }
            if (ok && leader) mma_commit(&bar_done);
            if (leader) mma_quiesce(&bar_quiet, p.st, 29);
        }
    } else {
        // ------------------------------------------------------------ gradient warpgroups (thread = key)
        const int wg = (warp - 2) >> 2;
        const int par = wg % kBwdParities, half = wg / kBwdParities;
        const int sub = warp & 3;
        const int row = sub * 32 + lane;
        const int gk = k0 + row;
        const uint32_t lane_base = tmem + ((uint32_t)(sub * 32) << 16);
        constexpr int CW = C::CW;
        const float g_uni = uniform_g(p);
        static_assert(kBwdParities == 1 && C::THREADS == 32 + kNbCount,
                      "every gradient warp takes part in every tile's named barriers");
        bool ok = true;
        for (int t = par; t < n_qt; t += kBwdParities) {
            const int s = t % C::NSTAGE, n = t / C::NSTAGE, buf = t & 1;
            const int q0 = (first_qt + t) * C::BM;
            const int ssid = t + 2 < n_qt ? nb_ssfree(t) : -1;   // the MMA warp waits only when it has a tile t+2
            if (ok)
                ok = __all_sync(0xffffffffu, mbar_wait(&bar_sfull[buf], (t >> 1) & 1, p.st, abort_v, 16) &&
                                                 mbar_wait(&bar_qfull[s], n & 1, p.st, abort_v, 17));
            if (!ok) {
                // The barriers the MMA warp waits on, without the work.  These
                // wait too (bar.sync), so that a warp here stays in step with the
                // MMA warp (the ids go round four tiles: see nb_dsfull).
                if (ssid >= 0) named_sync(ssid, kNbCount);
                named_sync(nb_dsfull(t), kNbCount);
                continue;
            }
            tc_fence_after();
            const float *ktab = reinterpret_cast<const float *>(sQ + s * C::STAGE_BYTES + C::GK) + half * CW;
            const float *gtab = ktab + C::BM, *ltab = gtab + C::BM, *stab = ltab + C::BM;
            const int qmin = gk - off - q0;        // first visible query column (causal)
            const uint32_t col = lane_base + buf * 128 + half * CW;   // this warpgroup's chunk
            const bool masked = p.causal && (k0 + C::BN - 1 > q0 + half * CW + off);
            const NamedRel rel{ssid};
            if (masked) {
                if (p.dkl)
                    dkv_chunk<TEACHER, true, true, CW, kBwdPiece, NamedRel, true>(
                        col, col + 64, p.ct, p.cs, ktab, gtab, 0.f, qmin - half * CW, rel, kNbCount, ltab, stab);
                else
                    dkv_chunk<TEACHER, true, false, CW, kBwdPiece, NamedRel, true>(
                        col, col + 64, p.ct, p.cs, ktab, gtab, g_uni, qmin - half * CW, rel, kNbCount, ltab, stab);
            } else {
                if (p.dkl)
                    dkv_chunk<TEACHER, false, true, CW, kBwdPiece, NamedRel, true>(
                        col, col + 64, p.ct, p.cs, ktab, gtab, 0.f, 0, rel, kNbCount, ltab, stab);
                else
                    dkv_chunk<TEACHER, false, false, CW, kBwdPiece, NamedRel, true>(
                        col, col + 64, p.ct, p.cs, ktab, gtab, g_uni, 0, rel, kNbCount, ltab, stab);
            }
            tmem_st_wait();
            tc_fence_before();
            named_arrive(nb_dsfull(t), kNbCount);
        }
        if (ok && n_qt > 0 && mbar_wait(&bar_done, 0, p.st, abort_v, 19)) {
            tc_fence_after();
            // every MMA and TMA copy is done: the stage ring is free for staging
            float *stage = reinterpret_cast<float *>(sQ) + (warp - 2) * 32 * (32 + kDrainPad);
            const int row0 = k0 + sub * 32;
            const int nvalid = max(0, min(32, p.N_K - row0));
            const size_t r0 = (size_t)bh * p.N_K + row0;
            constexpr int HS = DS / C::NWG, HT = DT / C::NWG;
            const float gs = p.dkl ? 1.f : g_uni;         // a uniform g was left out of dS
            // a padding key: its row is zero (the length is read again here rather
            // than kept live through the tile loop)
            const bool pad = PAD && gk >= key_count(p.kv_len, bh / p.H, p.N_K, nullptr, false);
            const size_t nk_all = (size_t)p.BH * p.N_K;   // rows of the output (or its per-head partial)
            drain_rows<HS>(lane_base + C::TMEM_DKS + wg * HS, p.out_s * gs, p.dk_s + r0 * DS + wg * HS, DS, nvalid,
                           stage, lane, pad, p.dk_s + nk_all * DS, p.st.word);
            if (TEACHER)
                drain_rows<HT>(lane_base + C::TMEM_DKT + wg * HT, p.out_t * gs, p.dk_t + r0 * DT + wg * HT, DT,
                               nvalid, stage, lane, pad, p.dk_t + nk_all * DT, p.st.word);
        } else if (n_qt == 0 && gk < p.N_K && wg == 0) {
            const size_t r = (size_t)bh * p.N_K + gk;
            if (bound_ok(r < (size_t)p.BH * p.N_K, p.st.word, kSiteZero)) {
                for (int c = 0; c < DS; ++c) p.dk_s[r * DS + c] = 0.f;
                if (TEACHER) for (int c = 0; c < DT; ++c) p.dk_t[r * DT + c] = 0.f;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

template <int DT, int DS, bool TEACHER>
__global__ void __launch_bounds__(DkvCfg<DT, DS, TEACHER>::THREADS, 1)
    streamkl_bwd_dkv_persistent_kernel(const __grid_constant__ CUtensorMap mQt, const __grid_constant__ CUtensorMap mKt,
                            const __grid_constant__ CUtensorMap mQs, const __grid_constant__ CUtensorMap mKs,
                            const BwdParams p) {
    // Persistent form of streamkl_bwd_dkv_kernel: each CTA works through its
    // items (128 keys of one head each, see persistent_item) one after the
    // other.  Tiles are counted across
    // items, so the Q stage ring, the logit buffers and their barriers simply
    // continue from one item to the next: the next item's Q stages load while
    // the last tiles of the current one are computed, its resident K rows
    // (already in shared memory by TMA when K_STAGED) go to tensor memory as
    // soon as the current item's last logit MMA has completed, and
    // its first logits are computed while the gradient warps write out the
    // current item's dK.
    using C = DkvCfg<DT, DS, TEACHER>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sKt = smem;
    uint8_t *sKs = sKt + C::KT_BYTES;
    uint8_t *sOnes = sKs + C::KS_BYTES;            // rank-1 MMA operand (1, 1, 1, 0, ...)
    uint8_t *sKst = sOnes + C::ONES_BYTES;         // K_TMEM: staging area of the next item's K rows
    uint8_t *sQ = sKst + C::KST_BYTES;             // stages: Q_t, Q_s, bias_t, bias_s, {g, KL}

    __shared__ uint64_t bar_qfull[C::NSTAGE], bar_qempty[C::NSTAGE], bar_sfull[2], bar_dsfull[2];
    __shared__ uint64_t bar_ssfree[2];             // all warps have read the buffer's student logits
    __shared__ uint64_t bar_k;                     // this item's resident K rows are in place
    __shared__ uint64_t bar_kfree;                 // the item's last logit MMA has completed
    __shared__ uint64_t bar_done;                  // the item's last gradient MMA has completed
    __shared__ uint64_t bar_quiet;                 // the MMA thread's issued MMAs have completed
    __shared__ uint64_t bar_kst, bar_kstfree;      // K_TMEM: staged K rows landed / copied out
    __shared__ uint32_t tmem_base_sh;
    __shared__ int abort_flag;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // tensors behind the four maps (bounds-checked build)
    const MapDims mdQt{DT, p.N_Q, p.BH}, mdQs{DS, p.N_Q, p.BH};
    const MapDims mdKt{DT, p.N_K, p.BH / p.H * p.Hkt}, mdKs{DS, p.N_K, p.BH / p.H * p.Hks};
    const int off = p.N_K - p.N_Q;
    const int n_qt_all = (p.N_Q + C::BM - 1) / C::BM;
    const int n_items = p.BH * p.n_tiles;
    // item j: key tile j / BH (low key tiles see the most queries), head j % BH;
    // an item whose keys are all padding has no visible pair (zero dK rows)
    auto item_geom = [&](int j, int &k0, int &bh, int &first_qt, int &n_qt) {
        k0 = (j / p.BH) * C::BN;
        bh = j % p.BH;
        first_qt = p.causal ? max(0, k0 - off) / C::BM : 0;
        n_qt = max(0, n_qt_all - first_qt);
        if (p.kv_len && k0 >= key_count(p.kv_len, bh / p.H, p.N_K, nullptr, false)) n_qt = 0;
    };

    if (warp == 0) {
        if (lane == 0) {
            for (int s = 0; s < C::NSTAGE; ++s) {
                mbar_init(&bar_qfull[s], 1 + 32);      // TMA expect_tx + every producer lane (constants)
                mbar_init(&bar_qempty[s], 1);
            }
            for (int b = 0; b < 2; ++b) {
                mbar_init(&bar_sfull[b], 1);
                mbar_init(&bar_dsfull[b], 4 * C::NH);
                mbar_init(&bar_ssfree[b], 4 * C::NH);
            }
            // K rows: one TMA arrival, or (in tensor memory) every gradient warp
            mbar_init(&bar_k, C::K_TMEM ? 4 * C::NH : 1);
            mbar_init(&bar_kfree, 1);
            mbar_init(&bar_done, 1);
            mbar_init(&bar_quiet, 1);
            mbar_init(&bar_kst, 1);
            mbar_init(&bar_kstfree, 4 * C::NH);
            abort_flag = 0;
            fence_barrier_init();
            prefetch_tmap(&mKt); prefetch_tmap(&mKs); prefetch_tmap(&mQt); prefetch_tmap(&mQs);
            // Start the first item's resident K tile and first Q stage right away,
            // so that their latency overlaps the set-up (the producer issues the
            // rest after it; issuing a TMA copy takes a while and the set-up
            // barrier waits for this thread).
            int k0, bh, first_qt, n_qt;
            item_geom(persistent_item(0, n_items), k0, bh, first_qt, n_qt);
            if (n_qt > 0) {
                const int bkt = key_head(bh, p.H, p.Hkt), bks = key_head(bh, p.H, p.Hks);
                if (!C::K_TMEM) {
                    mbar_expect_tx(&bar_k, C::KT_BYTES + C::KS_BYTES);
#pragma unroll
                    for (int b = 0; b < DT / 64; ++b) tma_load_3d(sKt + b * C::KBLK, &mKt, &bar_k, b * 64, k0, bkt, mdKt, p.st.word);
#pragma unroll
                    for (int b = 0; b < DS / 64; ++b) tma_load_3d(sKs + b * C::KBLK, &mKs, &bar_k, b * 64, k0, bks, mdKs, p.st.word);
                } else if (C::K_STAGED) {
                    mbar_expect_tx(&bar_kst, C::KST_BYTES);
#pragma unroll
                    for (int b = 0; b < DT / 64; ++b) tma_load_3d(sKst + b * C::KBLK, &mKt, &bar_kst, b * 64, k0, bkt, mdKt, p.st.word);
#pragma unroll
                    for (int b = 0; b < DS / 64; ++b)
                        tma_load_3d(sKst + C::BN * DT * 2 + b * C::KBLK, &mKs, &bar_kst, b * 64, k0, bks, mdKs, p.st.word);
                }
                mbar_expect_tx(&bar_qfull[0], C::STAGE_TMA);
#pragma unroll
                for (int b = 0; b < DT / 64; ++b)
                    tma_load_3d(sQ + b * C::QBLK, &mQt, &bar_qfull[0], b * 64, first_qt * C::BM, bh, mdQt, p.st.word);
#pragma unroll
                for (int b = 0; b < DS / 64; ++b)
                    tma_load_3d(sQ + C::QT_BYTES + b * C::QBLK, &mQs, &bar_qfull[0], b * 64, first_qt * C::BM, bh, mdQs, p.st.word);
            }
        }
    } else if (warp == 1) {
        tmem_alloc(&tmem_base_sh, 512);
        tmem_relinquish();
    }
    if (warp >= 2 && warp < 6) {
        // One warpgroup writes the constant MMA operands (and makes them
        // visible to the tensor core: the proxy fence is costly per warp).
        // Unswizzled K-major [rows][16] bf16 layout: row r, K block kb at
        // (r / 8) * 256 + kb * 128 + (r % 8) * 16.  The ones matrix has 1.0 in
        // K elements 0..2 of every row; the bias tiles start all zero and the
        // producer later writes only K elements 0..2 of each row.
        const int tid = threadIdx.x - 64;
        for (int i = tid; i < C::ONES_BYTES / 16; i += 128) {
            const bool first_block = ((i >> 3) & 1) == 0;   // 16-byte units: 8 rows per K block
            *reinterpret_cast<uint4 *>(sOnes + i * 16) =
                first_block ? make_uint4(0x3F803F80u, 0x00003F80u, 0u, 0u) : make_uint4(0u, 0u, 0u, 0u);
        }
        for (int st = 0; st < C::NSTAGE; ++st)
            for (int i = tid; i < 2 * C::BIAS_BYTES / 16; i += 128)
                *reinterpret_cast<uint4 *>(sQ + st * C::STAGE_BYTES + C::BIAS_T + i * 16) = make_uint4(0u, 0u, 0u, 0u);
        fence_proxy_async_smem();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base_sh;
    volatile int *abort_v = &abort_flag;

    if (warp == 0) {
        // ------------------------------------------------------------ producer (TMA + per-query constants)
        const float g_all = uniform_g(p);
        int issued = 0, k_issued = 0;              // Q stages and K tiles issued so far
        int g0 = 0;                                // this item's first tile, counted across items
        bool ok = true;
        // K_STAGED: the K rows of the items with tiles pass through the staging
        // area one item ahead; each copy is issued once the gradient warps have
        // copied the previous item's rows out of it (checked without blocking
        // at every Q stage, so the ring keeps filling meanwhile).  Lane 0 alone
        // keeps this state and issues the copies: no warp-wide step depends on
        // it, so lanes that leave the loop early on an abort cannot stall it.
        int kst_r = 0, kst_n = 0;                  // next item to stage: position, index among items with tiles
        int kst_k0 = 0, kst_bh = 0;
        bool kst_more = false;                     // such an item exists
        auto kst_find = [&]() {
            kst_more = false;
            for (;; ++kst_r) {
                const int jj = persistent_item(kst_r, n_items);
                if (jj < 0) return;
                int fq, nq;
                item_geom(jj, kst_k0, kst_bh, fq, nq);
                if (nq > 0) { kst_more = true; return; }
            }
        };
        auto kst_issue = [&](bool block) -> bool {     // lane 0 only
            if (!C::K_STAGED || !kst_more) return true;
            if (kst_n > 0 && !mbar_try_wait(&bar_kstfree, (kst_n - 1) & 1)) {
                if (!block) return true;
                if (!mbar_wait(&bar_kstfree, (kst_n - 1) & 1, p.st, abort_v, 20)) return false;
            }
            mbar_expect_tx(&bar_kst, C::KST_BYTES);
            const int kbt = key_head(kst_bh, p.H, p.Hkt), kbs = key_head(kst_bh, p.H, p.Hks);
#pragma unroll
            for (int b = 0; b < DT / 64; ++b)
                tma_load_3d(sKst + b * C::KBLK, &mKt, &bar_kst, b * 64, kst_k0, kbt, mdKt, p.st.word);
#pragma unroll
            for (int b = 0; b < DS / 64; ++b)
                tma_load_3d(sKst + C::BN * DT * 2 + b * C::KBLK, &mKs, &bar_kst, b * 64, kst_k0, kbs, mdKs, p.st.word);
            ++kst_n;
            ++kst_r;
            kst_find();
            return true;
        };
        if (C::K_STAGED && lane == 0) {
            kst_find();
            if (kst_more && kst_r == 0) {          // the first item's rows were issued during set-up
                ++kst_n;
                ++kst_r;
                kst_find();
            }
        }
        for (int r = 0, it = 0; ok; ++r) {
            const int j = persistent_item(r, n_items);
            if (j < 0) break;
            int k0, bh, first_qt, n_qt;
            item_geom(j, k0, bh, first_qt, n_qt);
            if (n_qt == 0) continue;
            // item 0 (when it has tiles): its K tile and first Q stage were issued during set-up
            const bool pre = r == 0;
            if (!C::K_TMEM && !pre) {
                // the previous item's K rows stay until its last logit MMA has completed
                if (it > 0 && !mbar_wait(&bar_kfree, (it - 1) & 1, p.st, abort_v, 10)) break;
                if (lane == 0) {
                    mbar_expect_tx(&bar_k, C::KT_BYTES + C::KS_BYTES);
                    const int bkt = key_head(bh, p.H, p.Hkt), bks = key_head(bh, p.H, p.Hks);
#pragma unroll
                    for (int b = 0; b < DT / 64; ++b) tma_load_3d(sKt + b * C::KBLK, &mKt, &bar_k, b * 64, k0, bkt, mdKt, p.st.word);
#pragma unroll
                    for (int b = 0; b < DS / 64; ++b) tma_load_3d(sKs + b * C::KBLK, &mKs, &bar_k, b * 64, k0, bks, mdKs, p.st.word);
                }
            }
            if (!C::K_TMEM) ++k_issued;
            if (C::K_TMEM && !C::K_STAGED && lane == 0) {
                // the next item's K rows, which the gradient warps copy into tensor
                // memory from global memory at this item's end: bring them into L2 now
                const int jn = persistent_item(r + 1, n_items);
                if (jn >= 0) {
                    int k0n, bhn, fqn, nqn;
                    item_geom(jn, k0n, bhn, fqn, nqn);
                    const int rows = min(C::BN, p.N_K - k0n);
                    const size_t bt = (size_t)key_head(bhn, p.H, p.Hkt) * p.N_K + k0n;
                    const size_t bs = (size_t)key_head(bhn, p.H, p.Hks) * p.N_K + k0n;
                    prefetch_l2(static_cast<const __nv_bfloat16 *>(p.kt_raw) + bt * DT, (uint32_t)rows * DT * 2);
                    prefetch_l2(static_cast<const __nv_bfloat16 *>(p.ks_raw) + bs * DS, (uint32_t)rows * DS * 2);
                }
            }
            // Per-query constants of a tile: lane l handles queries l and l + 32.
            // They are fetched from global memory two tiles ahead into registers,
            // with loads the compiler may not move (ld_now), so that their latency
            // overlaps the tiles in between instead of stalling the ring.
            auto load_consts = [&](int t, float4 (&v)[2]) {   // raw {lse_t, lse_s, g, kl}
                const int q0 = (first_qt + t) * C::BM;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int i = q0 + lane + 32 * h;
                    v[h] = make_float4(0.f, 0.f, 0.f, 0.f);        // rows past N_Q: g = 0, so dS = 0
                    if (t < n_qt && i < p.N_Q && bound_ok(bh < p.BH && i >= 0, p.st.word, kSiteConst)) {
                        const size_t rr = (size_t)bh * p.N_Q + i;
                        v[h].x = ld_now(p.lse_t + rr);
                        v[h].y = ld_now(p.lse_s + rr);
                        v[h].z = p.dkl ? ld_now(p.dkl + rr) : g_all;
                        v[h].w = ld_now(p.kl + rr);
                    }
                }
            };
            float4 c0[2], c1[2], c2[2];
            load_consts(0, c1);
            load_consts(1, c2);
            for (int t = 0; t < n_qt; ++t) {
                const int gg = g0 + t, s = gg % C::NSTAGE, n = gg / C::NSTAGE;
                const int q0 = (first_qt + t) * C::BM;
                c0[0] = c1[0]; c0[1] = c1[1];
                c1[0] = c2[0]; c1[1] = c2[1];
                load_consts(t + 2, c2);
                if (n > 0 && !mbar_wait(&bar_qempty[s], (n - 1) & 1, p.st, abort_v, 11)) { ok = false; break; }
                if (lane == 0) kst_issue(false);
                uint8_t *st = sQ + s * C::STAGE_BYTES;
                if (lane == 0 && !(pre && t == 0)) {
                    mbar_expect_tx(&bar_qfull[s], C::STAGE_TMA);
#pragma unroll
                    for (int b = 0; b < DT / 64; ++b)
                        tma_load_3d(st + b * C::QBLK, &mQt, &bar_qfull[s], b * 64, q0, bh, mdQt, p.st.word);
#pragma unroll
                    for (int b = 0; b < DS / 64; ++b)
                        tma_load_3d(st + C::QT_BYTES + b * C::QBLK, &mQs, &bar_qfull[s], b * 64, q0, bh, mdQs, p.st.word);
                }
                float *ktab = reinterpret_cast<float *>(st + C::GK), *gtab = ktab + C::BM;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int q = lane + 32 * h;
                    ktab[q] = c0[h].w * kLog2eF;
                    gtab[q] = c0[h].z;
                    const uint32_t row = (uint32_t)(q >> 3) * 256u + (uint32_t)(q & 7) * 16u;
                    *reinterpret_cast<uint2 *>(st + C::BIAS_T + row) = split3_bf16(-c0[h].x * p.inv_scale_t);
                    *reinterpret_cast<uint2 *>(st + C::BIAS_S + row) = split3_bf16(-c0[h].y * p.inv_scale_s);
                }
                fence_proxy_async_smem();          // the bias rows are read by the tensor core
                mbar_arrive(&bar_qfull[s]);
                issued = gg + 1;
            }
            g0 += n_qt;
            ++it;
        }
        if (lane == 0)
            while (ok && kst_more)
                if (!kst_issue(true)) ok = false;
        if (*abort_v && lane == 0) {
            // let the copies in flight land before the CTA's memory is released
            DevStatus quick = p.st;
            quick.budget_ns = 50000000ull;
            volatile int never = 0;
            if (k_issued > 0) mbar_wait(&bar_k, (k_issued - 1) & 1, quick, &never, 11);
            if (kst_n > 0) mbar_wait(&bar_kst, (kst_n - 1) & 1, quick, &never, 11);
            for (int t = (issued > C::NSTAGE ? issued - C::NSTAGE : 0); t < issued; ++t)
                mbar_wait(&bar_qfull[t % C::NSTAGE], (t / C::NSTAGE) & 1, quick, &never, 11);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        // Descriptors are built once (warp-uniform) and advanced by constant offsets.
        const uint64_t dKt = sw128_desc(smem_u32(sKt), 16, 1024), dKs = sw128_desc(smem_u32(sKs), 16, 1024);
        const uint64_t dQ0 = sw128_desc(smem_u32(sQ), 16, 1024);          // K-major view of a stage
        const uint64_t dQ0mn = sw128_desc(smem_u32(sQ), C::QBLK, 1024);   // MN-major view of a stage
        const uint64_t dOnes = plain_desc(smem_u32(sOnes), 128, 256);
        const uint64_t dBias0 = plain_desc(smem_u32(sQ + C::BIAS_T), 128, 256);
        if (elect_one()) {
            // Student S^T of tile gg (plus its rank-1 bias -LSE_s / scale_s) into
            // columns [64, 128) of buffer gg & 1, once the tile's Q stage has landed.
            auto issue_ss = [&](int gg) -> bool {
                const int s = gg % C::NSTAGE, n = gg / C::NSTAGE, buf = gg & 1;
                if (!mbar_wait(&bar_qfull[s], n & 1, p.st, abort_v, 12)) return false;
                tc_fence_after();
                const uint64_t dQs = desc_add(dQ0, s * C::STAGE_BYTES + C::QT_BYTES);
                const uint64_t dBs = desc_add(dBias0, s * C::STAGE_BYTES + C::BIAS_BYTES);
#pragma unroll
                for (int kk = 0; kk < DS / 16; ++kk) {
                    const uint64_t b = desc_add(dQs, (kk >> 2) * C::QBLK + (kk & 3) * 32);
                    if constexpr (C::K_TMEM)
                        mma_bf16_ts(tmem + buf * 128 + 64, tmem + C::TMEM_KS + kk * 8, b, C::IDESC_S, kk > 0);
                    else
                        mma_bf16_ss(tmem + buf * 128 + 64, desc_add(dKs, (kk >> 2) * C::KBLK + (kk & 3) * 32), b,
                                    C::IDESC_S, kk > 0);
                }
                mma_bf16_ss(tmem + buf * 128 + 64, dOnes, dBs, C::IDESC_S, 1);
                return true;
            };
            // Teacher S^T (plus bias) into columns [0, 64), then signal the tile;
            // after an item's last logits, signal that its K rows may go.
            auto issue_st = [&](int gg, bool last) {
                const int s = gg % C::NSTAGE, buf = gg & 1;
                const uint64_t dQt = desc_add(dQ0, s * C::STAGE_BYTES);
                const uint64_t dBt = desc_add(dBias0, s * C::STAGE_BYTES);
#pragma unroll
                for (int kk = 0; kk < DT / 16; ++kk) {
                    const uint64_t b = desc_add(dQt, (kk >> 2) * C::QBLK + (kk & 3) * 32);
                    if constexpr (C::K_TMEM)
                        mma_bf16_ts(tmem + buf * 128, tmem + C::TMEM_KT + kk * 8, b, C::IDESC_S, kk > 0);
                    else
                        mma_bf16_ss(tmem + buf * 128, desc_add(dKt, (kk >> 2) * C::KBLK + (kk & 3) * 32), b,
                                    C::IDESC_S, kk > 0);
                }
                mma_bf16_ss(tmem + buf * 128, dOnes, dBt, C::IDESC_S, 1);
                mma_commit(&bar_sfull[buf]);
                if (last) mma_commit(&bar_kfree);
            };
            bool ok = true;
            int g0 = 0;
            for (int r = 0, it = 0; ok; ++r) {
                const int j = persistent_item(r, n_items);
                if (j < 0) break;
                int k0, bh, first_qt, n_qt;
                item_geom(j, k0, bh, first_qt, n_qt);
                if (n_qt == 0) continue;
                if (!mbar_wait(&bar_k, it & 1, p.st, abort_v, 14)) break;
                // the item's first two tiles; their buffers were last used by the
                // previous item's last two tiles, whose student logits every warp
                // must have read (their dS is consumed by MMAs issued earlier)
                for (int t = 0; t < 2 && t < n_qt; ++t) {
                    const int gg = g0 + t;
                    if (gg >= 2 && !mbar_wait(&bar_ssfree[gg & 1], ((gg - 2) >> 1) & 1, p.st, abort_v, 13)) {
                        ok = false;
                        break;
                    }
                    if (!issue_ss(gg)) { ok = false; break; }
                    issue_st(gg, t == n_qt - 1);
                }
                for (int t = 0; ok && t < n_qt; ++t) {
                    const int gg = g0 + t, buf = gg & 1, s = gg % C::NSTAGE;
                    const bool next = t + 2 < n_qt;
                    // The student logits of tile t+2 go into this buffer as soon as every
                    // warp has read tile t's (they keep their dS in the teacher half).
                    if (next && (!mbar_wait(&bar_ssfree[buf], (gg >> 1) & 1, p.st, abort_v, 13) || !issue_ss(gg + 2)))
                        break;
                    if (!mbar_wait(&bar_dsfull[buf], (gg >> 1) & 1, p.st, abort_v, 15)) break;
                    tc_fence_after();
                    const uint64_t mQt = desc_add(dQ0mn, s * C::STAGE_BYTES), mQs = desc_add(mQt, C::QT_BYTES);
                    // dK_s += dS_s^T Q_s : A = dS_s^T from TMEM (buffer columns [0,32)), B = Q_s (MN-major)
#pragma unroll
                    for (int ks = 0; ks < C::BM / 16; ++ks)
                        mma_bf16_ts(tmem + C::TMEM_DKS, tmem + buf * 128 + ds_col_s(ks), desc_add(mQs, ks * 2048),
                                    C::IDESC_KS, (t > 0 || ks > 0));
                    if (TEACHER) {
#pragma unroll
                        for (int ks = 0; ks < C::BM / 16; ++ks)
                            mma_bf16_ts(tmem + C::TMEM_DKT, tmem + buf * 128 + ds_col_t(ks), desc_add(mQt, ks * 2048),
                                        C::IDESC_KT, (t > 0 || ks > 0));
                    }
                    mma_commit(&bar_qempty[s]);
                    if (next) issue_st(gg + 2, t + 2 == n_qt - 1);
                }
                if (!ok || *abort_v) break;
                mma_commit(&bar_done);
                g0 += n_qt;
                ++it;
            }
            mma_quiesce(&bar_quiet, p.st, 29);
        }
    } else {
        // ------------------------------------------------------------ gradient warpgroups (thread = key)
        const int wg = (warp - 2) >> 2;
        const int half = wg;
        const int sub = warp & 3;
        const int row = sub * 32 + lane;
        const uint32_t lane_base = tmem + ((uint32_t)(sub * 32) << 16);
        constexpr int CW = C::CW;
        const float g_uni = uniform_g(p);
        const float gs = p.dkl ? 1.f : g_uni;             // a uniform g was left out of dS
        bool ok = true;
        int g0 = 0;
        // K rows of the item into tensor memory (K_TMEM), once the previous
        // item's last logit MMA has completed
        auto k_to_tmem = [&](int it, int k0, int bh) -> bool {
            if (it > 0 && !mbar_wait(&bar_kfree, (it - 1) & 1, p.st, abort_v, 18)) return false;
            if constexpr (C::K_STAGED) {
                if (!mbar_wait(&bar_kst, it & 1, p.st, abort_v, 21)) return false;
                tc_fence_after();
                tile_rows_to_tmem<DT>(lane_base + C::TMEM_KT, sKst, wg, row);
                tile_rows_to_tmem<DS>(lane_base + C::TMEM_KS, sKst + C::BN * DT * 2, wg, row);
            } else {
                tc_fence_after();
                resident_to_tmem<DT>(tmem, C::TMEM_KT, p.kt_raw, key_head(bh, p.H, p.Hkt), p.N_K, k0, wg, sub, lane, mdKt.n2, p.st.word);
                resident_to_tmem<DS>(tmem, C::TMEM_KS, p.ks_raw, key_head(bh, p.H, p.Hks), p.N_K, k0, wg, sub, lane, mdKs.n2, p.st.word);
            }
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if (C::K_STAGED) mbar_arrive(&bar_kstfree);
                mbar_arrive(&bar_k);
            }
            return true;
        };
        int it = 0;
        bool k_ready = false;                      // K_TMEM: this item's K rows already copied
        for (int r = 0; ok; ++r) {
            const int j = persistent_item(r, n_items);
            if (j < 0) break;
            int k0, bh, first_qt, n_qt;
            item_geom(j, k0, bh, first_qt, n_qt);
            const int gk = k0 + row;
            if (n_qt == 0) {
                if (gk < p.N_K && wg == 0) {       // no visible query: dK = 0
                    const size_t rr = (size_t)bh * p.N_K + gk;
                    if (bound_ok(rr < (size_t)p.BH * p.N_K, p.st.word, kSiteZero)) {
                        for (int c = 0; c < DS; ++c) p.dk_s[rr * DS + c] = 0.f;
                        if (TEACHER) for (int c = 0; c < DT; ++c) p.dk_t[rr * DT + c] = 0.f;
                    }
                }
            } else {
                if (C::K_TMEM && !k_ready && !k_to_tmem(it, k0, bh)) { ok = false; break; }
                k_ready = false;
                for (int t = 0; t < n_qt; ++t) {
                    const int gg = g0 + t, s = gg % C::NSTAGE, n = gg / C::NSTAGE, buf = gg & 1;
                    const int q0 = (first_qt + t) * C::BM;
                    if (!mbar_wait(&bar_sfull[buf], (gg >> 1) & 1, p.st, abort_v, 16) ||
                        !mbar_wait(&bar_qfull[s], n & 1, p.st, abort_v, 17)) { ok = false; break; }
                    tc_fence_after();
                    const float *ktab = reinterpret_cast<const float *>(sQ + s * C::STAGE_BYTES + C::GK) + half * CW;
                    const float *gtab = ktab + C::BM;
                    const int qmin = gk - off - q0;        // first visible query column (causal)
                    const uint32_t col = lane_base + buf * 128 + half * CW;   // this warpgroup's chunk
                    const bool masked = p.causal && (k0 + C::BN - 1 > q0 + half * CW + off);
                    uint64_t *sfree = &bar_ssfree[buf];
                    if (masked) {
                        if (p.dkl)
                            dkv_chunk<TEACHER, true, true, CW>(col, col + 64, p.ct, p.cs, ktab, gtab, 0.f,
                                                               qmin - half * CW, sfree, 0);
                        else
                            dkv_chunk<TEACHER, true, false, CW>(col, col + 64, p.ct, p.cs, ktab, gtab, g_uni,
                                                                qmin - half * CW, sfree, 0);
                    } else {
                        if (p.dkl) dkv_chunk<TEACHER, false, true, CW>(col, col + 64, p.ct, p.cs, ktab, gtab, 0.f, 0, sfree, 0);
                        else dkv_chunk<TEACHER, false, false, CW>(col, col + 64, p.ct, p.cs, ktab, gtab, g_uni, 0, sfree, 0);
                    }
                    tmem_st_wait();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&bar_dsfull[buf]);
                }
                if (!ok) break;
                if constexpr (C::K_TMEM) {
                    // the next item with tiles: its K rows go to tensor memory as soon
                    // as this item's logits are done
                    for (int rn = r + 1;; ++rn) {
                        const int jn = persistent_item(rn, n_items);
                        if (jn < 0) break;
                        int k0n, bhn, fqn, nqn;
                        item_geom(jn, k0n, bhn, fqn, nqn);
                        if (nqn == 0) continue;
                        if (!k_to_tmem(it + 1, k0n, bhn)) ok = false;
                        k_ready = true;
                        break;
                    }
                    if (!ok) break;
                }
                if (!mbar_wait(&bar_done, it & 1, p.st, abort_v, 19)) { ok = false; break; }
                tc_fence_after();
                // dK rows straight from tensor memory to global memory (the stage
                // ring already holds the next item's tiles)
                const bool valid = gk < p.N_K;
                const bool pad = gk >= key_count(p.kv_len, bh / p.H, p.N_K, nullptr, false);   // zero row
                const size_t grow = (size_t)bh * p.N_K + gk;
                constexpr int HS = DS / C::NWG, HT = DT / C::NWG;
                const size_t nk_all = (size_t)p.BH * p.N_K;   // rows of the output (or its per-head partial)
                drain_row<HS>(lane_base + C::TMEM_DKS + wg * HS, p.out_s * gs, p.dk_s + grow * DS + wg * HS, valid,
                              pad, p.dk_s + nk_all * DS, p.st.word);
                if (TEACHER)
                    drain_row<HT>(lane_base + C::TMEM_DKT + wg * HT, p.out_t * gs, p.dk_t + grow * DT + wg * HT, valid,
                                  pad, p.dk_t + nk_all * DT, p.st.word);
                tc_fence_before();
                g0 += n_qt;
                ++it;
            }
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
    // Tensor memory: logit buffers [0, 256), dQ_s, dQ_t, and, when they fit
    // (Q_TMEM: the student-only and d = 64 cases), this CTA's Q_t and Q_s rows
    // as packed bf16, so the logit MMAs read only the K tile from shared memory.
    static constexpr uint32_t TMEM_DQS = 256, TMEM_DQT = 256 + DS;
    static constexpr uint32_t TMEM_QT = TMEM_DQT + (TEACHER ? DT : 0), TMEM_QS = TMEM_QT + DT / 2;
    static constexpr bool Q_TMEM = TMEM_QS + DS / 2 <= 512;
    // Hand-off of each tile between the gradient warps and the MMA warp through
    // named barriers where the logit MMAs read Q from shared memory; through
    // mbarriers (polled by the MMA thread) where Q sits in tensor memory, the
    // form in which the named barriers measured slower.
    static constexpr bool NAMED = !Q_TMEM;
    static constexpr int QT_BYTES = Q_TMEM ? 0 : BM * DT * 2, QS_BYTES = Q_TMEM ? 0 : BM * DS * 2;
    static constexpr int KT_BYTES = BN * DT * 2, KS_BYTES = BN * DS * 2;
    static constexpr int STAGE_BYTES = KT_BYTES + KS_BYTES;
    static constexpr int FIXED = QT_BYTES + QS_BYTES;
    static constexpr int NS_RAW = (224 * 1024 - FIXED) / STAGE_BYTES;
    static constexpr int NSTAGE = NS_RAW < 2 ? 2 : (NS_RAW > 6 ? 6 : NS_RAW);
    // the student logits of tile t+2 are issued before the gradient MMA of
    // tile t releases its stage, so t+2 must not need that stage
    static_assert(NSTAGE >= 3, "stage ring too shallow for the early student logits");
    static_assert(NSTAGE * STAGE_BYTES >= 16 * 32 * (32 + kDrainPad) * 4, "stage ring doubles as the drain staging area");
    static constexpr int SMEM = FIXED + NSTAGE * STAGE_BYTES + 1024;
    static constexpr int NH = kBwdHalves, NWG = kBwdParities * kBwdHalves, CW = BN / NH;
    static constexpr int THREADS = 64 + 128 * NWG;
    static constexpr uint32_t IDESC_S = idesc_bf16(128, BN, 0, 0);
    static constexpr uint32_t IDESC_QS = idesc_bf16(128, DS, 0, 1);
    static constexpr uint32_t IDESC_QT = idesc_bf16(128, DT, 0, 1);
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
    uint8_t *sK = sQs + C::QS_BYTES;               // stages: K_t, K_s

    __shared__ uint64_t bar_q, bar_kfull[C::NSTAGE], bar_kempty[C::NSTAGE], bar_sfull[2], bar_dsfull[2];
    __shared__ uint64_t bar_ssfree[2];             // all warps have read the buffer's student logits
    __shared__ uint64_t bar_done;
    __shared__ uint64_t bar_quiet;                 // the MMA thread's issued MMAs have completed
    __shared__ uint32_t tmem_base_sh;
    __shared__ int abort_flag;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // tensors behind the four maps (bounds-checked build)
    const MapDims mdQt{DT, p.N_Q, p.BH}, mdQs{DS, p.N_Q, p.BH};
    const MapDims mdKt{DT, p.N_K, p.BH / p.H * p.Hkt}, mdKs{DS, p.N_K, p.BH / p.H * p.Hks};
    // heaviest causal query tiles first; the key splits of a tile are adjacent
    const int lin = (int)(blockIdx.x / p.BH);
    const int split = lin % p.splits;
    const int qt_idx = p.n_tiles - 1 - lin / p.splits;
    const int bh = (int)(blockIdx.x % p.BH);
    const int q0 = qt_idx * C::BM;
    const int off = p.N_K - p.N_Q;
    // this head's key heads, and its keys that are not padding
    const int bkt = key_head(bh, p.H, p.Hkt), bks = key_head(bh, p.H, p.Hks);
    const int nk = key_count(p.kv_len, bh / p.H, p.N_K, p.st.word, false);
    int kend = nk;
    if (p.causal) kend = min(nk, min(q0 + C::BM - 1, p.N_Q - 1) + off + 1);
    const int n_all = (kend + C::BN - 1) / C::BN;
    // this CTA's key tiles [kt_lo, kt_lo + n_kt); loops count from 0.  With
    // padding a range may be empty (n_kt = 0): the CTA then writes zeros.
    const int kt_lo = (int)((long long)n_all * split / p.splits);
    const int n_kt = (int)((long long)n_all * (split + 1) / p.splits) - kt_lo;

    if (threadIdx.x == 0) {
        mbar_init(&bar_q, 1);
        for (int s = 0; s < C::NSTAGE; ++s) {
            mbar_init(&bar_kfull[s], 1);
            mbar_init(&bar_kempty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bar_sfull[b], 1);
            mbar_init(&bar_dsfull[b], 4 * C::NH);
            mbar_init(&bar_ssfree[b], 4 * C::NH);
        }
        mbar_init(&bar_done, 1);
        mbar_init(&bar_quiet, 1);
        abort_flag = 0;
        fence_barrier_init();
        // Start the resident Q tile and the first K stage right away, so that
        // their latency overlaps the set-up.  Issuing a TMA copy takes a while
        // and the set-up barrier waits for this thread, so the producer issues
        // the other stages after it.
        prefetch_tmap(&mKt); prefetch_tmap(&mKs);
        if (!C::Q_TMEM) {
            prefetch_tmap(&mQt); prefetch_tmap(&mQs);
            mbar_expect_tx(&bar_q, C::QT_BYTES + C::QS_BYTES);
#pragma unroll
            for (int b = 0; b < DT / 64; ++b) tma_load_3d(sQt + b * C::QBLK, &mQt, &bar_q, b * 64, q0, bh, mdQt, p.st.word);
#pragma unroll
            for (int b = 0; b < DS / 64; ++b) tma_load_3d(sQs + b * C::QBLK, &mQs, &bar_q, b * 64, q0, bh, mdQs, p.st.word);
        }
        if (n_kt > 0) {
            mbar_expect_tx(&bar_kfull[0], C::STAGE_BYTES);
#pragma unroll
            for (int b = 0; b < DT / 64; ++b)
                tma_load_3d(sK + b * C::KBLK, &mKt, &bar_kfull[0], b * 64, kt_lo * C::BN, bkt, mdKt, p.st.word);
#pragma unroll
            for (int b = 0; b < DS / 64; ++b)
                tma_load_3d(sK + C::KT_BYTES + b * C::KBLK, &mKs, &bar_kfull[0], b * 64, kt_lo * C::BN, bks, mdKs, p.st.word);
        }
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
    if constexpr (C::Q_TMEM) {
        if (warp >= 2) {
            const int wg = (warp - 2) >> 2, sub = warp & 3;
            resident_to_tmem<DT>(tmem, C::TMEM_QT, p.qt_raw, bh, p.N_Q, q0, wg, sub, lane, mdQt.n2, p.st.word);
            resident_to_tmem<DS>(tmem, C::TMEM_QS, p.qs_raw, bh, p.N_Q, q0, wg, sub, lane, mdQs.n2, p.st.word);
            tmem_st_wait();
        }
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    }

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (elect_one()) {
            // Q and the first key tile were issued during set-up
            int issued = min(1, n_kt);
            for (int kt = issued; kt < n_kt; ++kt) {
                const int s = kt % C::NSTAGE, n = kt / C::NSTAGE;
                if (n > 0 && !mbar_wait(&bar_kempty[s], (n - 1) & 1, p.st, abort_v, 21)) break;
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
                DevStatus quick = p.st;
                quick.budget_ns = 50000000ull;
                volatile int never = 0;
                if (!C::Q_TMEM) mbar_wait(&bar_q, 0, quick, &never, 21);
                for (int kt = (issued > C::NSTAGE ? issued - C::NSTAGE : 0); kt < issued; ++kt)
                    mbar_wait(&bar_kfull[kt % C::NSTAGE], (kt / C::NSTAGE) & 1, quick, &never, 21);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        // Descriptors are built once (warp-uniform) and advanced by constant offsets.
        const uint64_t dQt = sw128_desc(smem_u32(sQt), 16, 1024), dQs = sw128_desc(smem_u32(sQs), 16, 1024);
        const uint64_t dK0 = sw128_desc(smem_u32(sK), 16, 1024);          // K-major view of a stage
        const uint64_t dK0mn = sw128_desc(smem_u32(sK), C::KBLK, 1024);   // MN-major view of a stage
        const bool leader = elect_one();
        const int leader_lane = __ffs(__ballot_sync(0xffffffffu, leader)) - 1;
        {
            // Student S of key tile kt into columns [64, 128) of buffer kt & 1,
            // once the tile's K stage has landed.
            auto issue_ss = [&](int kt) -> bool {
                const int s = kt % C::NSTAGE, n = kt / C::NSTAGE, buf = kt & 1;
                if (!mbar_wait(&bar_kfull[s], n & 1, p.st, abort_v, 22)) return false;
                tc_fence_after();
                const uint64_t dKs = desc_add(dK0, s * C::STAGE_BYTES + C::KT_BYTES);
#pragma unroll
                for (int kk = 0; kk < DS / 16; ++kk) {
                    const uint64_t b = desc_add(dKs, (kk >> 2) * C::KBLK + (kk & 3) * 32);
                    if constexpr (C::Q_TMEM)
                        mma_bf16_ts(tmem + buf * 128 + 64, tmem + C::TMEM_QS + kk * 8, b, C::IDESC_S, kk > 0);
                    else
                        mma_bf16_ss(tmem + buf * 128 + 64, desc_add(dQs, (kk >> 2) * C::QBLK + (kk & 3) * 32), b,
                                    C::IDESC_S, kk > 0);
                }
                return true;
            };
            // Teacher S into columns [0, 64), then signal the tile.
            auto issue_st = [&](int kt) {
                const int s = kt % C::NSTAGE, buf = kt & 1;
                const uint64_t dKt = desc_add(dK0, s * C::STAGE_BYTES);
#pragma unroll
                for (int kk = 0; kk < DT / 16; ++kk) {
                    const uint64_t b = desc_add(dKt, (kk >> 2) * C::KBLK + (kk & 3) * 32);
                    if constexpr (C::Q_TMEM)
                        mma_bf16_ts(tmem + buf * 128, tmem + C::TMEM_QT + kk * 8, b, C::IDESC_S, kk > 0);
                    else
                        mma_bf16_ss(tmem + buf * 128, desc_add(dQt, (kk >> 2) * C::QBLK + (kk & 3) * 32), b,
                                    C::IDESC_S, kk > 0);
                }
                mma_commit(&bar_sfull[buf]);
            };
            // dQ += dS K for tile kt (A = dS from TMEM, buffer columns [0, 32) for
            // the student, B = the K stage, MN-major), then release the stage.
            auto issue_dq = [&](int kt) {
                const int s = kt % C::NSTAGE, buf = kt & 1;
                const uint64_t mKt = desc_add(dK0mn, s * C::STAGE_BYTES), mKs = desc_add(mKt, C::KT_BYTES);
#pragma unroll
                for (int ks = 0; ks < C::BN / 16; ++ks)
                    mma_bf16_ts(tmem + C::TMEM_DQS, tmem + buf * 128 + ds_col_s(ks), desc_add(mKs, ks * 2048),
                                C::IDESC_QS, (kt > 0 || ks > 0));
                if (TEACHER) {
#pragma unroll
                    for (int ks = 0; ks < C::BN / 16; ++ks)
                        mma_bf16_ts(tmem + C::TMEM_DQT, tmem + buf * 128 + ds_col_t(ks), desc_add(mKt, ks * 2048),
                                    C::IDESC_QT, (kt > 0 || ks > 0));
                }
                mma_commit(&bar_kempty[s]);
            };
            bool ok = true;
            if (leader) {
                ok = C::Q_TMEM || mbar_wait(&bar_q, 0, p.st, abort_v, 24);
                for (int kt = 0; ok && kt < 2 && kt < n_kt; ++kt) {
                    ok = issue_ss(kt);
                    if (ok) issue_st(kt);
                }
            }
            if constexpr (C::NAMED) {
                ok = __shfl_sync(0xffffffffu, ok, leader_lane);
                // The whole warp takes part in the named barriers; after a failed
                // wait it keeps taking part (issuing nothing), so that the gradient
                // warps, which make the same arrivals in any case, never wait on it.
                for (int kt = 0; kt < n_kt; ++kt) {
                    // tile kt hands off on nb_ssfree(kt) and nb_dsfull(kt)
                    const bool next = kt + 2 < n_kt;
                    // the student logits of tile kt+2 go into this buffer as soon as
                    // every warp has read tile kt's (they keep their dS in the teacher half)
                    __syncwarp();
                    if (next) named_sync(nb_ssfree(kt), kNbCount);
                    if (ok && next) {
                        tc_fence_after();
                        bool r = true;
                        if (leader) r = issue_ss(kt + 2);
                        ok = __shfl_sync(0xffffffffu, r, leader_lane);
                    }
                    named_sync(nb_dsfull(kt), kNbCount);
                    if (ok && leader) {
                        tc_fence_after();
                        issue_dq(kt);
                        if (next) issue_st(kt + 2);
                    }
                    __syncwarp();
                }
                if (ok && leader) mma_commit(&bar_done);
            } else if (leader) {
                for (int kt = 0; ok && kt < n_kt; ++kt) {
                    const int buf = kt & 1;
                    const bool next = kt + 2 < n_kt;
                    if (next && (!mbar_wait(&bar_ssfree[buf], (kt >> 1) & 1, p.st, abort_v, 23) || !issue_ss(kt + 2)))
                        break;
                    if (!mbar_wait(&bar_dsfull[buf], (kt >> 1) & 1, p.st, abort_v, 25)) break;
                    tc_fence_after();
                    issue_dq(kt);
                    if (next) issue_st(kt + 2);
                }
                mma_commit(&bar_done);
            }
            if (leader) mma_quiesce(&bar_quiet, p.st, 29);
        }
    } else {
        // ------------------------------------------------------------ gradient warpgroups (thread = query)
        const int wg = (warp - 2) >> 2;
        const int par = wg % kBwdParities, half = wg / kBwdParities;
        const int sub = warp & 3;
        const int gq = q0 + sub * 32 + lane;
        const uint32_t lane_base = tmem + ((uint32_t)(sub * 32) << 16);
        constexpr int CW = C::CW;
        float Lt = 0.f, Ls = 0.f, g = 0.f, KL2 = 0.f;
        if (gq < p.N_Q) {
            const size_t r = (size_t)bh * p.N_Q + gq;
            Lt = p.lse_t[r] * kLog2eF;
            Ls = p.lse_s[r] * kLog2eF;
            g = p.dkl ? p.dkl[r] : uniform_g(p);
            KL2 = p.kl[r] * kLog2eF;
        }
        const int lim = p.causal ? min(nk, gq + off + 1) : nk;   // first hidden key
        static_assert(kBwdParities == 1 && C::THREADS == 32 + kNbCount,
                      "every gradient warp takes part in every tile's hand-off");
        bool ok = true;
        for (int kt = par; kt < n_kt; kt += kBwdParities) {
            const int buf = kt & 1;
            const int ssid = kt + 2 < n_kt ? nb_ssfree(kt) : -1;   // the MMA warp waits only when it has a tile t+2
            if constexpr (C::NAMED) {
                if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&bar_sfull[buf], (kt >> 1) & 1, p.st, abort_v, 26));
                if (!ok) {
                    // The barriers the MMA warp waits on, without the work.  These
                    // wait too (bar.sync), so that a warp here stays in step with the
                    // MMA warp (the ids go round four tiles: see nb_dsfull).
                    if (ssid >= 0) named_sync(ssid, kNbCount);
                    named_sync(nb_dsfull(kt), kNbCount);
                    continue;
                }
            } else {
                if (!mbar_wait(&bar_sfull[buf], (kt >> 1) & 1, p.st, abort_v, 26)) { ok = false; break; }
            }
            tc_fence_after();
            const auto rel = [&] {
                if constexpr (C::NAMED) return NamedRel{ssid};
                else return &bar_ssfree[buf];
            }();
            const uint32_t col = lane_base + buf * 128 + half * CW;   // this warpgroup's chunk
            const int kb = (kt_lo + kt) * C::BN + half * CW;
            const bool masked = (kb + CW > nk) || (p.causal && (kb + CW - 1 > q0 + off));
            if (masked)
                dq_chunk<TEACHER, true, CW>(col, col + 64, p.ct, p.cs, Lt, Ls, g, KL2, kb, lim, rel, kNbCount);
            else
                dq_chunk<TEACHER, false, CW>(col, col + 64, p.ct, p.cs, Lt, Ls, g, KL2, kb, lim, rel, kNbCount);
            tmem_st_wait();
            tc_fence_before();
            if constexpr (C::NAMED) {
                named_arrive(nb_dsfull(kt), kNbCount);
            } else {
                __syncwarp();
                if (lane == 0) mbar_arrive(&bar_dsfull[buf]);
            }
        }
        if (ok && mbar_wait(&bar_done, 0, p.st, abort_v, 28)) {
            tc_fence_after();
            // every MMA and TMA copy is done: the stage ring is free for staging
            float *stage = reinterpret_cast<float *>(sK) + (warp - 2) * 32 * (32 + kDrainPad);
            const int row0 = q0 + sub * 32;
            const int nvalid = max(0, min(32, p.N_Q - row0));
            size_t r0 = (size_t)bh * p.N_Q + row0;
            float *dst_s = p.dq_s, *dst_t = p.dq_t;
            if (p.splits > 1) {             // this split's partial, summed by streamkl_split_sum_kernel
                r0 += (size_t)split * p.BH * p.N_Q;
                dst_s = p.part_s;
                dst_t = p.part_t;
            }
            constexpr int HS = DS / C::NWG, HT = DT / C::NWG;
            // the row's g was left out of dS; no key tile: nothing was accumulated
            const size_t nq_all = (size_t)p.splits * p.BH * p.N_Q;   // rows of the output, or of all partials
            drain_rows<HS>(lane_base + C::TMEM_DQS + wg * HS, p.out_s * g, dst_s + r0 * DS + wg * HS, DS, nvalid,
                           stage, lane, n_kt == 0, dst_s + (p.splits > 1 ? nq_all : (size_t)p.BH * p.N_Q) * DS,
                           p.st.word);
            if (TEACHER)
                drain_rows<HT>(lane_base + C::TMEM_DQT + wg * HT, p.out_t * g, dst_t + r0 * DT + wg * HT, DT, nvalid,
                               stage, lane, n_kt == 0,
                               dst_t + (p.splits > 1 ? nq_all : (size_t)p.BH * p.N_Q) * DT, p.st.word);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// Grouped key heads: the key-owner kernel writes one dK partial per query head
// ([B, H, N_K, d]); a key head's gradient is the sum of its group's partials,
// out[b, g] = sum over u = 0 .. G-1 of part[b, g G + u], in that order
// (deterministic).  nd = N_K * d, a multiple of 4; 16-byte aligned arrays.
__global__ void __launch_bounds__(256) streamkl_group_sum_kernel(const float *__restrict__ part, int H, int Hk,
                                                                 long long nd, long long n_out,
                                                                 float *__restrict__ out) {
    const int G = H / Hk;
    const long long nd4 = nd >> 2;
    const float4 *p4 = reinterpret_cast<const float4 *>(part);
    float4 *o4 = reinterpret_cast<float4 *>(out);
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < (n_out >> 2);
         i += (long long)gridDim.x * blockDim.x) {
        const long long bg = i / nd4, e = i - bg * nd4;          // key head b * Hk + g, element
        const long long first = (bg / Hk) * H + (bg % Hk) * G;   // its group's first query head
        float4 a = __ldg(p4 + first * nd4 + e);
        for (int u = 1; u < G; ++u) {
            const float4 b = __ldg(p4 + (first + u) * nd4 + e);
            a.x += b.x; a.y += b.y; a.z += b.z; a.w += b.w;
        }
        o4[i] = a;
    }
}

// out[i] = sum over s of part[s * n + i], s in order (deterministic); n % 4 == 0
// and 16-byte aligned arrays (gradient rows are 64 or 128 floats).
__global__ void __launch_bounds__(256) streamkl_split_sum_kernel(const float *__restrict__ part, int splits,
                                                                 long long n, float *__restrict__ out) {
    const long long n4 = n >> 2;
    const float4 *p4 = reinterpret_cast<const float4 *>(part);
    float4 *o4 = reinterpret_cast<float4 *>(out);
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += (long long)gridDim.x * blockDim.x) {
        float4 a = __ldg(p4 + i);
        for (int s = 1; s < splits; ++s) {
            const float4 b = __ldg(p4 + (long long)s * n4 + i);
            a.x += b.x; a.y += b.y; a.z += b.z; a.w += b.w;
        }
        o4[i] = a;
    }
}

}  // namespace skl
