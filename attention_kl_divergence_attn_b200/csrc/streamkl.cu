// streamkl.cu — the C ABI declared in include/streamkl.h: argument checks,
// TMA descriptor set-up and kernel launches.  No entry point allocates device
// memory, synchronises (except streamkl_check) or aborts.
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <algorithm>
#include <set>
#include <utility>
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>

#include "streamkl.h"
#include "sm100.cuh"
#include "fwd.cuh"
#include "bwd.cuh"

using namespace skl;

namespace {

constexpr size_t kWorkspaceBytes = 256;
constexpr unsigned long long kWaitBudgetNs = 2000000000ull;   // 2 s per bounded wait
constexpr float kLog2e = 1.4426950408889634074f;

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// 3-D map over a [BH, N, d] bf16 tensor: box = 64 columns x `rows` rows x 1
// head, 128-byte swizzle, zero fill outside [0,N) so ragged tiles read zeros.
bool make_map(CUtensorMap *m, const void *ptr, int d, int N, int BH, int rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)N, (cuuint64_t)BH};
    cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)N * d * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)rows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

streamkl_status check_device() {
    int dev = 0, major = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return STREAMKL_ERR_CUDA;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
        return STREAMKL_ERR_CUDA;
    return major == 10 ? STREAMKL_OK : STREAMKL_ERR_UNSUPPORTED;
}

streamkl_status check_shape(int B, int H, int N_Q, int N_K, int d_t, int d_s, int causal, float scale_t,
                            float scale_s) {
    if (B < 0 || H < 0 || N_Q < 0 || N_K < 0) return STREAMKL_ERR_INVALID_ARG;
    if (causal != 0 && causal != 1) return STREAMKL_ERR_INVALID_ARG;
    if (causal && N_Q > N_K) return STREAMKL_ERR_INVALID_ARG;
    if (!causal && N_K == 0 && N_Q > 0 && B > 0 && H > 0) return STREAMKL_ERR_INVALID_ARG;
    if (!(scale_t > 0.f) || !(scale_s > 0.f) || scale_t == INFINITY || scale_s == INFINITY)
        return STREAMKL_ERR_INVALID_ARG;
    if ((long long)B * H > (1ll << 24) || N_Q > (1 << 24) || N_K > (1 << 24)) return STREAMKL_ERR_INVALID_ARG;
    if ((d_t != 64 && d_t != 128) || (d_s != 64 && d_s != 128)) return STREAMKL_ERR_UNSUPPORTED;
    return STREAMKL_OK;
}

// Grouped key heads and padding: K_t, K_s have H_kt, H_ks heads, each at
// least 1 and dividing H; the key lengths (if any) are 4-byte aligned ints.
streamkl_status check_heads(int H, int H_kt, int H_ks, const int *kv_len) {
    if (H_kt < 1 || H_ks < 1 || H_kt > (1 << 24) || H_ks > (1 << 24)) return STREAMKL_ERR_INVALID_ARG;
    if (H > 0 && (H % H_kt != 0 || H % H_ks != 0)) return STREAMKL_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(kv_len) & 3u) != 0) return STREAMKL_ERR_INVALID_ARG;
    return STREAMKL_OK;
}

// Input and output pointers of the forward: required (and 16-byte aligned)
// unless the problem has no rows.  Makes no CUDA call.
streamkl_status fwd_check_pointers(const void *q_t, const void *k_t, const void *q_s, const void *k_s, int B, int H,
                                   int N_Q, const float *kl, const float *lse_t, const float *lse_s) {
    if ((long long)B * H * N_Q == 0) return STREAMKL_OK;
    if (!q_t || !k_t || !q_s || !k_s || !kl || !lse_t || !lse_s) return STREAMKL_ERR_INVALID_ARG;
    if (!aligned16(q_t) || !aligned16(k_t) || !aligned16(q_s) || !aligned16(k_s)) return STREAMKL_ERR_INVALID_ARG;
    return STREAMKL_OK;
}

// Raises a kernel's dynamic shared-memory limit once per (kernel, device)
// (the attribute persists), so that later calls, including calls made while a
// stream is being captured into a CUDA graph, only launch.
std::mutex g_attr_mutex;
std::set<std::pair<const void *, int>> g_attr_done;

template <typename K>
cudaError_t set_smem(K kernel, int bytes) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorUnknown;
    const std::pair<const void *, int> key(reinterpret_cast<const void *>(kernel), dev);
    std::lock_guard<std::mutex> lock(g_attr_mutex);
    if (g_attr_done.count(key)) return cudaSuccess;
    const cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess) g_attr_done.insert(key);
    return e;
}

constexpr int kFwdWarpgroups = 4;

int sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return 0;
    return n;
}

// Key splits for the kernels that own 128-row query tiles and walk 64-key
// tiles (the forward and the query-owner backward).  With few query tiles
// (short N_Q, long N_K) one CTA per tile leaves SMs idle in the last wave, so
// each tile's key range is cut into S pieces that run as separate CTAs and
// are combined afterwards (forward: the associative merge of the online
// states; backward: a fixed-order sum of dQ partials).  S minimises
// waves(S) / S, the estimated time in units of one whole-row CTA, with 2 %
// added per extra piece for the combine pass and per-CTA set-up; every piece
// keeps at least kMinSplitTiles key tiles of the shortest (first, under
// causal) query tile.
constexpr int kMaxSplits = 32, kMinSplitTiles = 4;

int key_splits(int BH, int N_Q, int N_K, int causal) {
    const int sms = sm_count();
    const long long ctas = (long long)BH * ((N_Q + 127) / 128);
    if (sms <= 0 || ctas == 0 || ctas >= 8ll * sms) return 1;
    int kend = N_K;
    if (causal) kend = std::min(N_K, std::min(127, N_Q - 1) + (N_K - N_Q) + 1);
    const int smax = std::min(kMaxSplits, ((kend + 63) / 64) / kMinSplitTiles);
    int best = 1;
    double best_t = 1e300;
    for (int S = 1; S <= std::max(1, smax); ++S) {
        const double waves = (double)((ctas * S + sms - 1) / sms);
        const double t = waves / S * (1.0 + 0.02 * (S - 1));
        if (t < best_t * (1.0 - 1e-9)) { best = S; best_t = t; }
    }
    return best;
}

// Workspace bytes beyond the status word that S key splits need.
size_t fwd_split_bytes(int S, long long rows) { return S > 1 ? (size_t)5 * S * rows * sizeof(float) : 0; }
size_t dq_split_bytes(int S, long long rows, int d_s, int d_t) {
    return S > 1 ? (size_t)S * rows * (d_s + d_t) * sizeof(float) : 0;
}

#ifndef STREAMKL_FWD_PERSISTENT
#define STREAMKL_FWD_PERSISTENT 1
#endif
// The forward runs persistent (one CTA per SM working through the query
// tiles, see streamkl_fwd_persistent_kernel).
constexpr bool kFwdPersistent = STREAMKL_FWD_PERSISTENT != 0;

template <int DT, int DS>
streamkl_status launch_fwd(const CUtensorMap &qt, const CUtensorMap &kt, const CUtensorMap &qs,
                           const CUtensorMap &ks, const FwdParams &p, cudaStream_t stream) {
    using C = FwdCfg<DT, DS, kFwdWarpgroups>;
    const long long items = (long long)p.BH * p.n_qt * p.splits;
    if constexpr (kFwdPersistent) {
        auto kern = streamkl_fwd_persistent_kernel<DT, DS, kFwdWarpgroups>;
        if (set_smem(kern, C::SMEM) != cudaSuccess) return STREAMKL_ERR_CUDA;
        const long long grid = std::min<long long>(items, std::max(1, sm_count()));
        kern<<<(unsigned)grid, C::THREADS, C::SMEM, stream>>>(qt, kt, qs, ks, p);
    } else {
        auto kern = streamkl_fwd_kernel<DT, DS, kFwdWarpgroups>;
        if (set_smem(kern, C::SMEM) != cudaSuccess) return STREAMKL_ERR_CUDA;
        kern<<<(unsigned)items, C::THREADS, C::SMEM, stream>>>(qt, kt, qs, ks, p);
    }
    if (cudaGetLastError() != cudaSuccess) return STREAMKL_ERR_CUDA;
    if (p.splits > 1) {
        const long long rows = (long long)p.BH * p.N_Q;
        streamkl_fwd_merge_kernel<<<(unsigned)((rows + 255) / 256), 256, 0, stream>>>(p.part, p.splits, rows, p.kl,
                                                                                      p.lse_t, p.lse_s);
        if (cudaGetLastError() != cudaSuccess) return STREAMKL_ERR_CUDA;
    }
    return STREAMKL_OK;
}

// Which backward kernels a call launches.
enum BwdParts { kPartDK = 1, kPartDQ = 2 };

// Where the key-owner kernel's dK goes when key heads are grouped: it writes
// one partial per query head to the workspace (p.dk_s / p.dk_t point there),
// and a fixed-order group sum writes each key head's gradient to these.
struct DkOut {
    float *dk_s, *dk_t;
};

streamkl_status group_sum(const float *part, int H, int Hk, int BK, int N_K, int d, float *out, cudaStream_t s) {
    const long long nd = (long long)N_K * d, n_out = (long long)BK * nd;
    const long long blocks = std::min<long long>((n_out / 4 + 255) / 256, 8ll * std::max(1, sm_count()));
    streamkl_group_sum_kernel<<<(unsigned)std::max(1ll, blocks), 256, 0, s>>>(part, H, Hk, nd, n_out, out);
    return cudaGetLastError() == cudaSuccess ? STREAMKL_OK : STREAMKL_ERR_CUDA;
}

template <int DT, int DS, bool TEACHER>
streamkl_status launch_bwd(const void *q_t, const void *k_t, const void *q_s, const void *k_s, int N_Q, int N_K,
                           BwdParams p, int parts, DkOut out, cudaStream_t stream) {
    using CK = DkvCfg<DT, DS, TEACHER>;
    using CQ = DqCfg<DT, DS, TEACHER>;
    const int BH = p.BH;
    const int BKt = BH / p.H * p.Hkt, BKs = BH / p.H * p.Hks;   // key heads of K_t, K_s
    CUtensorMap mqt, mkt, mqs, mks;
    if (parts & kPartDK) {
        // key-owner kernel: K boxes of 128 rows, Q boxes of 64 rows
        if (!make_map(&mqt, q_t, DT, N_Q, BH, CK::BM) || !make_map(&mkt, k_t, DT, N_K, BKt, CK::BN) ||
            !make_map(&mqs, q_s, DS, N_Q, BH, CK::BM) || !make_map(&mks, k_s, DS, N_K, BKs, CK::BN))
            return STREAMKL_ERR_CUDA;
        p.n_tiles = (N_K + CK::BN - 1) / CK::BN;
        const long long items = (long long)BH * p.n_tiles;
        // When the K rows live in tensor memory the kernel has registers to spare
        // and the persistent form (one CTA per SM working through its share of
        // the items, overlapping each item's start with the previous one's end)
        // is faster; at the register limit (teacher and student K in shared
        // memory) one CTA per item keeps the inner loop faster.
        if constexpr (CK::K_TMEM) {
            auto kdkv = streamkl_bwd_dkv_persistent_kernel<DT, DS, TEACHER>;
            if (set_smem(kdkv, CK::SMEM) != cudaSuccess) return STREAMKL_ERR_CUDA;
            const long long grid = std::min<long long>(items, std::max(1, sm_count()));
            kdkv<<<(unsigned)grid, CK::THREADS, CK::SMEM, stream>>>(mqt, mkt, mqs, mks, p);
        } else {
            auto kdkv = p.kv_len ? streamkl_bwd_dkv_kernel<DT, DS, TEACHER, true>
                                 : streamkl_bwd_dkv_kernel<DT, DS, TEACHER, false>;
            if (set_smem(kdkv, CK::SMEM) != cudaSuccess) return STREAMKL_ERR_CUDA;
            kdkv<<<(unsigned)items, CK::THREADS, CK::SMEM, stream>>>(mqt, mkt, mqs, mks, p);
        }
        if (cudaGetLastError() != cudaSuccess) return STREAMKL_ERR_CUDA;
        // grouped key heads: each key head's gradient is its group's partials summed in order
        streamkl_status st = STREAMKL_OK;
        if (out.dk_s != p.dk_s && (st = group_sum(p.dk_s, p.H, p.Hks, BKs, N_K, DS, out.dk_s, stream)) != STREAMKL_OK)
            return st;
        if (TEACHER && out.dk_t != p.dk_t &&
            (st = group_sum(p.dk_t, p.H, p.Hkt, BKt, N_K, DT, out.dk_t, stream)) != STREAMKL_OK)
            return st;
    }
    if (parts & kPartDQ) {
        // query-owner kernel: Q boxes of 128 rows, K boxes of 64 rows
        if (!make_map(&mqt, q_t, DT, N_Q, BH, CQ::BM) || !make_map(&mkt, k_t, DT, N_K, BKt, CQ::BN) ||
            !make_map(&mqs, q_s, DS, N_Q, BH, CQ::BM) || !make_map(&mks, k_s, DS, N_K, BKs, CQ::BN))
            return STREAMKL_ERR_CUDA;
        auto kdq = streamkl_bwd_dq_kernel<DT, DS, TEACHER>;
        if (set_smem(kdq, CQ::SMEM) != cudaSuccess) return STREAMKL_ERR_CUDA;
        p.n_tiles = (N_Q + CQ::BM - 1) / CQ::BM;
        kdq<<<(unsigned)((long long)BH * p.n_tiles * p.splits), CQ::THREADS, CQ::SMEM, stream>>>(mqt, mkt, mqs,
                                                                                              mks, p);
        if (cudaGetLastError() != cudaSuccess) return STREAMKL_ERR_CUDA;
        if (p.splits > 1) {
            const long long rows = (long long)BH * N_Q;
            const int sms = std::max(1, sm_count());
            for (int side = 0; side < (TEACHER ? 2 : 1); ++side) {
                const long long n = rows * (side ? DT : DS);
                const long long blocks = std::min<long long>((n / 4 + 255) / 256, 8ll * sms);
                streamkl_split_sum_kernel<<<(unsigned)blocks, 256, 0, stream>>>(side ? p.part_t : p.part_s, p.splits,
                                                                                 n, side ? p.dq_t : p.dq_s);
                if (cudaGetLastError() != cudaSuccess) return STREAMKL_ERR_CUDA;
            }
        }
    }
    return STREAMKL_OK;
}

template <bool TEACHER>
streamkl_status dispatch_bwd(int d_t, int d_s, const void *q_t, const void *k_t, const void *q_s, const void *k_s,
                             int N_Q, int N_K, const BwdParams &p, int parts, DkOut out, cudaStream_t s) {
    if (d_t == 64 && d_s == 64) return launch_bwd<64, 64, TEACHER>(q_t, k_t, q_s, k_s, N_Q, N_K, p, parts, out, s);
    if (d_t == 128 && d_s == 128) return launch_bwd<128, 128, TEACHER>(q_t, k_t, q_s, k_s, N_Q, N_K, p, parts, out, s);
    if (d_t == 128 && d_s == 64) return launch_bwd<128, 64, TEACHER>(q_t, k_t, q_s, k_s, N_Q, N_K, p, parts, out, s);
    return launch_bwd<64, 128, TEACHER>(q_t, k_t, q_s, k_s, N_Q, N_K, p, parts, out, s);
}

// Bytes of workspace beyond the status word that the key-owner kernel needs
// for its per-query-head dK partials when key heads are grouped (required).
size_t dk_group_bytes(long long BH, int N_K, int d_t, int d_s, int H, int H_kt, int H_ks, bool teacher) {
    size_t n = 0;
    if (H_ks < H) n += (size_t)BH * N_K * d_s;
    if (teacher && H_kt < H) n += (size_t)BH * N_K * d_t;
    return n * sizeof(float);
}

// Shared body of the backward entry points.  `parts` selects the kernels; the
// gradient pointers a part does not write may be NULL.  K_t and K_s have
// H_kt, H_ks heads (dividing H); kv_len (per batch, nullable) marks padding.
streamkl_status bwd_common(const void *q_t, const void *k_t, const void *q_s, const void *k_s, int B, int H,
                           int H_kt, int H_ks, int N_Q, int N_K, int d_t, int d_s, float scale_t, float scale_s,
                           int causal, const int *kv_len, const float *kl, const float *lse_t, const float *lse_s,
                           const float *dkl, float dloss, const float *dloss_dev, float *dq_s, float *dk_s,
                           float *dq_t, float *dk_t, void *workspace, size_t workspace_bytes, void *stream,
                           int parts) {
    streamkl_status st = check_shape(B, H, N_Q, N_K, d_t, d_s, causal, scale_t, scale_s);
    if (st != STREAMKL_OK) return st;
    if ((st = check_heads(H, H_kt, H_ks, kv_len)) != STREAMKL_OK) return st;
    if (!workspace || workspace_bytes < kWorkspaceBytes) return STREAMKL_ERR_WORKSPACE;
    if (!aligned16(workspace)) return STREAMKL_ERR_INVALID_ARG;
    const bool want_dk = parts & kPartDK, want_dq = parts & kPartDQ;
    if (!(dloss == dloss)) return STREAMKL_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    const int BH = B * H;
    const long long BKt = (long long)B * H_kt, BKs = (long long)B * H_ks;
    // Outputs with no elements may be NULL (an empty tensor has no storage).
    const bool dk_out = want_dk && (long long)BH * N_K > 0, dq_out = want_dq && (long long)BH * N_Q > 0;
    // the teacher pair of each part must be both given or both absent
    if (dk_out && dq_out && ((dq_t == nullptr) != (dk_t == nullptr))) return STREAMKL_ERR_INVALID_ARG;
    const bool teacher = dk_out ? dk_t != nullptr : dq_t != nullptr;
    if (dk_out && (!dk_s || (teacher && !dk_t))) return STREAMKL_ERR_INVALID_ARG;
    if (dq_out && (!dq_s || (teacher && !dq_t))) return STREAMKL_ERR_INVALID_ARG;
    const size_t dk_part = want_dk ? dk_group_bytes(BH, N_K, d_t, d_s, H, H_kt, H_ks, teacher) : 0;
    if (dk_part > 0 && workspace_bytes < kWorkspaceBytes + dk_part) return STREAMKL_ERR_WORKSPACE;
    if ((long long)BH * N_K == 0) return STREAMKL_OK;       // no keys (so no rows either): nothing to write
    if ((long long)BH * N_Q == 0) {                         // keys but no queries: every dK is zero
        if (want_dk) {
            if (cudaMemsetAsync(dk_s, 0, (size_t)BKs * N_K * d_s * sizeof(float), s) != cudaSuccess)
                return STREAMKL_ERR_CUDA;
            if (teacher && cudaMemsetAsync(dk_t, 0, (size_t)BKt * N_K * d_t * sizeof(float), s) != cudaSuccess)
                return STREAMKL_ERR_CUDA;
        }
        return STREAMKL_OK;
    }
    if (!q_t || !k_t || !q_s || !k_s || !kl || !lse_t || !lse_s) return STREAMKL_ERR_INVALID_ARG;
    if (!aligned16(q_t) || !aligned16(k_t) || !aligned16(q_s) || !aligned16(k_s)) return STREAMKL_ERR_INVALID_ARG;
    if (want_dk && (!aligned16(dk_s) || (teacher && !aligned16(dk_t)))) return STREAMKL_ERR_INVALID_ARG;
    if (want_dq && (!aligned16(dq_s) || (teacher && !aligned16(dq_t)))) return STREAMKL_ERR_INVALID_ARG;
    if ((st = check_device()) != STREAMKL_OK) return st;

    BwdParams p;
    memset(&p, 0, sizeof p);
    p.BH = BH; p.N_Q = N_Q; p.N_K = N_K; p.causal = causal;
    p.H = H; p.Hkt = H_kt; p.Hks = H_ks; p.kv_len = kv_len;
    p.ct = scale_t * kLog2e; p.cs = scale_s * kLog2e;
    p.out_t = scale_t * 0.69314718055994530942f;
    p.out_s = scale_s;
    p.kl = kl; p.lse_t = lse_t; p.lse_s = lse_s; p.dkl = dkl;
    if (dloss_dev) {                 // g = dloss (a scale) times the device scalar
        p.g_const = dloss;
        p.g_dev = dloss_dev;
    } else {
        p.g_const = (float)((double)dloss / ((double)BH * (double)N_Q));
    }
    p.inv_scale_t = 1.0f / scale_t;
    p.inv_scale_s = 1.0f / scale_s;
    p.dq_s = dq_s; p.dk_s = dk_s; p.dq_t = dq_t; p.dk_t = dk_t;
    DkOut out{dk_s, dk_t};
    if (dk_part > 0) {               // grouped key heads: per-query-head partials in the workspace
        float *part = reinterpret_cast<float *>(static_cast<char *>(workspace) + kWorkspaceBytes);
        if (H_ks < H) {
            p.dk_s = part;
            part += (size_t)BH * N_K * d_s;
        }
        if (teacher && H_kt < H) p.dk_t = part;
    }
    p.qt_raw = q_t; p.kt_raw = k_t; p.qs_raw = q_s; p.ks_raw = k_s;
    p.st.word = static_cast<uint32_t *>(workspace);
    p.st.budget_ns = kWaitBudgetNs;
    p.splits = 1;
    if (want_dq) {
        // dQ partials of key splits reuse the bytes after the status word: the
        // dK partials there are summed (same stream) before the dQ kernel runs
        const long long rows = (long long)BH * N_Q;
        const int S = key_splits(BH, N_Q, N_K, causal);
        if (S > 1 && workspace_bytes >= kWorkspaceBytes + dq_split_bytes(S, rows, d_s, teacher ? d_t : 0)) {
            p.splits = S;
            p.part_s = reinterpret_cast<float *>(static_cast<char *>(workspace) + kWorkspaceBytes);
            p.part_t = p.part_s + (size_t)S * rows * d_s;
        }
    }
    return teacher ? dispatch_bwd<true>(d_t, d_s, q_t, k_t, q_s, k_s, N_Q, N_K, p, parts, out, s)
                   : dispatch_bwd<false>(d_t, d_s, q_t, k_t, q_s, k_s, N_Q, N_K, p, parts, out, s);
}

// Shared body of the forward entry points.  K_t and K_s have H_kt, H_ks heads
// (dividing H); kv_len (per batch, nullable) marks padding.
streamkl_status fwd_common(const void *q_t, const void *k_t, const void *q_s, const void *k_s, int B, int H,
                           int H_kt, int H_ks, int N_Q, int N_K, int d_t, int d_s, float scale_t, float scale_s,
                           int causal, const int *kv_len, float *kl, float *lse_t, float *lse_s, float *loss_mean,
                           void *workspace, size_t workspace_bytes, void *stream) {
    streamkl_status st = check_shape(B, H, N_Q, N_K, d_t, d_s, causal, scale_t, scale_s);
    if (st != STREAMKL_OK) return st;
    if ((st = check_heads(H, H_kt, H_ks, kv_len)) != STREAMKL_OK) return st;
    if (!workspace || workspace_bytes < kWorkspaceBytes) return STREAMKL_ERR_WORKSPACE;
    if (!aligned16(workspace)) return STREAMKL_ERR_INVALID_ARG;
    if ((st = fwd_check_pointers(q_t, k_t, q_s, k_s, B, H, N_Q, kl, lse_t, lse_s)) != STREAMKL_OK) return st;
    cudaStream_t s = (cudaStream_t)stream;
    const int BH = B * H;
    const long long rows = (long long)BH * N_Q;
    if (rows == 0) {
        if (loss_mean) streamkl_mean_kernel<<<kMeanCtas, kMeanThreads, 0, s>>>(kl, 0, 1.0, 1.0, loss_mean);
        return cudaGetLastError() == cudaSuccess ? STREAMKL_OK : STREAMKL_ERR_CUDA;
    }
    if ((st = check_device()) != STREAMKL_OK) return st;

    CUtensorMap mqt, mkt, mqs, mks;
    // Q boxes of 128 rows (one query tile), K boxes of 64 rows (one key tile)
    if (!make_map(&mqt, q_t, d_t, N_Q, BH, 128) || !make_map(&mkt, k_t, d_t, N_K, B * H_kt, 64) ||
        !make_map(&mqs, q_s, d_s, N_Q, BH, 128) || !make_map(&mks, k_s, d_s, N_K, B * H_ks, 64))
        return STREAMKL_ERR_CUDA;
    FwdParams p;
    p.BH = BH; p.N_Q = N_Q; p.N_K = N_K; p.causal = causal;
    p.H = H; p.Hkt = H_kt; p.Hks = H_ks; p.kv_len = kv_len;
    p.n_qt = (N_Q + 127) / 128;
    p.ct = scale_t * kLog2e; p.cs = scale_s * kLog2e;
    p.kl = kl; p.lse_t = lse_t; p.lse_s = lse_s;
    p.st.word = static_cast<uint32_t *>(workspace);
    p.st.budget_ns = kWaitBudgetNs;
    p.splits = 1;
    p.part = nullptr;
    {
        const int S = key_splits(BH, N_Q, N_K, causal);
        if (S > 1 && workspace_bytes >= kWorkspaceBytes + fwd_split_bytes(S, rows)) {
            p.splits = S;
            p.part = reinterpret_cast<float *>(static_cast<char *>(workspace) + kWorkspaceBytes);
        }
    }
    if (d_t == 64 && d_s == 64) st = launch_fwd<64, 64>(mqt, mkt, mqs, mks, p, s);
    else if (d_t == 128 && d_s == 128) st = launch_fwd<128, 128>(mqt, mkt, mqs, mks, p, s);
    else if (d_t == 128 && d_s == 64) st = launch_fwd<128, 64>(mqt, mkt, mqs, mks, p, s);
    else st = launch_fwd<64, 128>(mqt, mkt, mqs, mks, p, s);
    if (st != STREAMKL_OK) return st;
    if (loss_mean) {
        streamkl_mean_kernel<<<kMeanCtas, kMeanThreads, 0, s>>>(kl, rows, (double)rows, 1.0, loss_mean);
        if (cudaGetLastError() != cudaSuccess) return STREAMKL_ERR_CUDA;
    }
    return STREAMKL_OK;
}

// Self-test of the failure path: one warp waits, with the library's bounded
// wait, on an mbarrier that nothing ever arrives at.  After `budget_ns` the
// wait records a timeout (who = kSelftestWho) in the status word, raises the
// CTA's abort flag (the other threads see it and return too) and the kernel
// ends normally, so the caller can check that the timeout is reported and that
// the CUDA context is still usable.  Nothing faults or hangs.
constexpr uint32_t kSelftestWho = 63;

__global__ void streamkl_selftest_timeout_kernel(DevStatus st) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();
    mbar_wait(&bar, 0, st, &abort_flag, kSelftestWho);
}

}  // namespace

extern "C" {

streamkl_status streamkl_selftest_timeout(void *workspace, size_t workspace_bytes, unsigned long long budget_ns,
                                          void *stream) {
    if (!workspace || workspace_bytes < kWorkspaceBytes) return STREAMKL_ERR_WORKSPACE;
    if (!aligned16(workspace)) return STREAMKL_ERR_INVALID_ARG;
    if (budget_ns < 1000000ull || budget_ns > kWaitBudgetNs) return STREAMKL_ERR_INVALID_ARG;
    streamkl_status st = check_device();
    if (st != STREAMKL_OK) return st;
    DevStatus ds;
    ds.word = static_cast<uint32_t *>(workspace);
    ds.budget_ns = budget_ns;
    streamkl_selftest_timeout_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(ds);
    return cudaGetLastError() == cudaSuccess ? STREAMKL_OK : STREAMKL_ERR_CUDA;
}

int streamkl_version(void) { return 100; }

size_t streamkl_workspace_size_ex(int B, int H, int H_kt, int H_ks, int N_Q, int N_K, int d_t, int d_s, int causal,
                                  int teacher_grads) {
    const size_t base = streamkl_workspace_size(B, H, N_Q, N_K, d_t, d_s, causal);
    if (B <= 0 || H <= 0 || N_K <= 0 || H_kt < 1 || H_ks < 1 || H % H_kt || H % H_ks) return base;
    if ((d_t != 64 && d_t != 128) || (d_s != 64 && d_s != 128)) return base;
    const size_t dk = dk_group_bytes((long long)B * H, N_K, d_t, d_s, H, H_kt, H_ks, teacher_grads != 0);
    const size_t need = kWorkspaceBytes + ((dk + 255) / 256) * 256;
    return std::max(base, need);
}

size_t streamkl_workspace_size(int B, int H, int N_Q, int N_K, int d_t, int d_s, int causal) {
    if (B <= 0 || H <= 0 || N_Q <= 0 || N_K <= 0 || (d_t != 64 && d_t != 128) || (d_s != 64 && d_s != 128))
        return kWorkspaceBytes;
    const long long rows = (long long)B * H * N_Q;
    const int S = key_splits(B * H, N_Q, N_K, causal ? 1 : 0);
    const size_t extra = std::max(fwd_split_bytes(S, rows), dq_split_bytes(S, rows, d_s, d_t));
    return kWorkspaceBytes + ((extra + 255) / 256) * 256;
}

const char *streamkl_strerror(streamkl_status s) {
    switch (s) {
        case STREAMKL_OK: return "ok";
        case STREAMKL_ERR_INVALID_ARG: return "invalid argument";
        case STREAMKL_ERR_UNSUPPORTED: return "unsupported problem or device";
        case STREAMKL_ERR_CUDA: return "CUDA error";
        case STREAMKL_ERR_TIMEOUT: return "a kernel gave up on a bounded wait";
        case STREAMKL_ERR_WORKSPACE: return "workspace missing or too small";
        case STREAMKL_ERR_BOUNDS: return "an access outside its tensor was skipped (bounds-checked build)";
    }
    return "unknown status";
}

streamkl_status streamkl_workspace_init(void *workspace, size_t workspace_bytes, void *stream) {
    if (!workspace) return STREAMKL_ERR_WORKSPACE;
    if (workspace_bytes < kWorkspaceBytes) return STREAMKL_ERR_WORKSPACE;
    return cudaMemsetAsync(workspace, 0, kWorkspaceBytes, (cudaStream_t)stream) == cudaSuccess ? STREAMKL_OK
                                                                                             : STREAMKL_ERR_CUDA;
}

streamkl_status streamkl_check(const void *workspace, void *stream, unsigned int *code_out) {
    cudaStream_t s = (cudaStream_t)stream;
    if (cudaStreamSynchronize(s) != cudaSuccess) return STREAMKL_ERR_CUDA;
    unsigned int word = 0;
    if (workspace) {
        if (cudaMemcpyAsync(&word, workspace, sizeof word, cudaMemcpyDeviceToHost, s) != cudaSuccess)
            return STREAMKL_ERR_CUDA;
        if (cudaMemsetAsync(const_cast<void *>(workspace), 0, sizeof word, s) != cudaSuccess)
            return STREAMKL_ERR_CUDA;
        if (cudaStreamSynchronize(s) != cudaSuccess) return STREAMKL_ERR_CUDA;
    }
    if (code_out) *code_out = word;
    if (cudaPeekAtLastError() != cudaSuccess) return STREAMKL_ERR_CUDA;
    if (word & kStatusTimeout) return STREAMKL_ERR_TIMEOUT;
    if (word & kStatusBounds) return STREAMKL_ERR_BOUNDS;
    return (word & kStatusBadLength) ? STREAMKL_ERR_INVALID_ARG : STREAMKL_OK;
}

streamkl_status streamkl_fwd(const void *q_t, const void *k_t, const void *q_s, const void *k_s, int B, int H,
                             int N_Q, int N_K, int d_t, int d_s, float scale_t, float scale_s, int causal,
                             float *kl, float *lse_t, float *lse_s, float *loss_mean, void *workspace,
                             size_t workspace_bytes, void *stream) {
    return fwd_common(q_t, k_t, q_s, k_s, B, H, H, H, N_Q, N_K, d_t, d_s, scale_t, scale_s, causal, nullptr, kl,
                      lse_t, lse_s, loss_mean, workspace, workspace_bytes, stream);
}

streamkl_status streamkl_fwd_ex(const void *q_t, const void *k_t, const void *q_s, const void *k_s, int B, int H,
                                int H_kt, int H_ks, int N_Q, int N_K, int d_t, int d_s, float scale_t, float scale_s,
                                int causal, const int *kv_len, float *kl, float *lse_t, float *lse_s,
                                float *loss_mean, void *workspace, size_t workspace_bytes, void *stream) {
    return fwd_common(q_t, k_t, q_s, k_s, B, H, H_kt, H_ks, N_Q, N_K, d_t, d_s, scale_t, scale_s, causal, kv_len, kl,
                      lse_t, lse_s, loss_mean, workspace, workspace_bytes, stream);
}



streamkl_status streamkl_bwd(const void *q_t, const void *k_t, const void *q_s, const void *k_s, int B, int H,
                             int N_Q, int N_K, int d_t, int d_s, float scale_t, float scale_s, int causal,
                             const float *kl, const float *lse_t, const float *lse_s, const float *dkl, float dloss,
                             float *dq_s, float *dk_s, float *dq_t, float *dk_t, void *workspace,
                             size_t workspace_bytes, void *stream) {
    return bwd_common(q_t, k_t, q_s, k_s, B, H, H, H, N_Q, N_K, d_t, d_s, scale_t, scale_s, causal, nullptr, kl, lse_t,
                      lse_s, dkl,
                      dloss, nullptr, dq_s, dk_s, dq_t, dk_t, workspace, workspace_bytes, stream, kPartDK | kPartDQ);
}

streamkl_status streamkl_bwd_dk(const void *q_t, const void *k_t, const void *q_s, const void *k_s, int B, int H,
                                int N_Q, int N_K, int d_t, int d_s, float scale_t, float scale_s, int causal,
                                const float *kl, const float *lse_t, const float *lse_s, const float *dkl,
                                float dloss, float *dk_s, float *dk_t, void *workspace, size_t workspace_bytes,
                                void *stream) {
    return bwd_common(q_t, k_t, q_s, k_s, B, H, H, H, N_Q, N_K, d_t, d_s, scale_t, scale_s, causal, nullptr, kl, lse_t,
                      lse_s, dkl,
                      dloss, nullptr, nullptr, dk_s, nullptr, dk_t, workspace, workspace_bytes, stream, kPartDK);
}

streamkl_status streamkl_bwd_dq(const void *q_t, const void *k_t, const void *q_s, const void *k_s, int B, int H,
                                int N_Q, int N_K, int d_t, int d_s, float scale_t, float scale_s, int causal,
                                const float *kl, const float *lse_t, const float *lse_s, const float *dkl,
                                float dloss, float *dq_s, float *dq_t, void *workspace, size_t workspace_bytes,
                                void *stream) {
    return bwd_common(q_t, k_t, q_s, k_s, B, H, H, H, N_Q, N_K, d_t, d_s, scale_t, scale_s, causal, nullptr, kl, lse_t,
                      lse_s, dkl,
                      dloss, nullptr, dq_s, nullptr, dq_t, nullptr, workspace, workspace_bytes, stream, kPartDQ);
}

streamkl_status streamkl_bwd_dloss_device(const void *q_t, const void *k_t, const void *q_s, const void *k_s, int B,
                                          int H, int N_Q, int N_K, int d_t, int d_s, float scale_t, float scale_s,
                                          int causal, const float *kl, const float *lse_t, const float *lse_s,
                                          const float *dkl, const float *dloss_dev, float dloss_scale, float *dq_s,
                                          float *dk_s, float *dq_t, float *dk_t, void *workspace,
                                          size_t workspace_bytes, void *stream) {
    if (!dkl && !dloss_dev) return STREAMKL_ERR_INVALID_ARG;
    return bwd_common(q_t, k_t, q_s, k_s, B, H, H, H, N_Q, N_K, d_t, d_s, scale_t, scale_s, causal, nullptr, kl, lse_t,
                      lse_s, dkl,
                      dloss_scale, dkl ? nullptr : dloss_dev, dq_s, dk_s, dq_t, dk_t, workspace, workspace_bytes,
                      stream, kPartDK | kPartDQ);
}

streamkl_status streamkl_bwd_ex(const void *q_t, const void *k_t, const void *q_s, const void *k_s, int B, int H,
                                int H_kt, int H_ks, int N_Q, int N_K, int d_t, int d_s, float scale_t, float scale_s,
                                int causal, const int *kv_len, const float *kl, const float *lse_t,
                                const float *lse_s, const float *dkl, float dloss, const float *dloss_dev,
                                float *dq_s, float *dk_s, float *dq_t, float *dk_t, int parts, void *workspace,
                                size_t workspace_bytes, void *stream) {
    if (parts < 1 || parts > (kPartDK | kPartDQ)) return STREAMKL_ERR_INVALID_ARG;
    // the part not asked for writes nothing: its pointers are ignored
    if (!(parts & kPartDK)) dk_s = dk_t = nullptr;
    if (!(parts & kPartDQ)) dq_s = dq_t = nullptr;
    return bwd_common(q_t, k_t, q_s, k_s, B, H, H_kt, H_ks, N_Q, N_K, d_t, d_s, scale_t, scale_s, causal, kv_len, kl,
                      lse_t, lse_s, dkl, dloss, dkl ? nullptr : dloss_dev, dq_s, dk_s, dq_t, dk_t, workspace,
                      workspace_bytes, stream, parts);
}

streamkl_status streamkl_loss_mean(const float *kl, long long n_rows, float *loss_mean, void *stream) {
    if (n_rows < 0 || !loss_mean || (n_rows > 0 && !kl)) return STREAMKL_ERR_INVALID_ARG;
    streamkl_mean_kernel<<<kMeanCtas, kMeanThreads, 0, (cudaStream_t)stream>>>(kl, n_rows, (double)n_rows, 1.0, loss_mean);
    return cudaGetLastError() == cudaSuccess ? STREAMKL_OK : STREAMKL_ERR_CUDA;
}

streamkl_status streamkl_loss_reduce(const float *kl, long long n_rows, double factor, float *out, void *stream) {
    if (n_rows < 0 || !out || (n_rows > 0 && !kl) || !(factor == factor)) return STREAMKL_ERR_INVALID_ARG;
    streamkl_mean_kernel<<<kMeanCtas, kMeanThreads, 0, (cudaStream_t)stream>>>(kl, n_rows, 1.0, factor, out);
    return cudaGetLastError() == cudaSuccess ? STREAMKL_OK : STREAMKL_ERR_CUDA;
}


}  // extern "C"

// ---------------------------------------------------------------------------
// Forward without any caller-provided device memory.
//
// Some callers cannot allocate device memory at all, not even the small
// workspace streamkl_fwd asks for: plug-in hosts that hand a library only the
// buffers they planned in advance, runtimes that forbid allocation once they
// are serving, and programs whose memory pool owns every byte of the device.
// For them the workspace (the device status word) lives in this file-scope
// array instead.  Every GPU that loads the library holds it until exit.
namespace {

constexpr size_t kNoAllocScratchBytes = 256;   // fixed maximum scratch of this entry point
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// The array's device address belongs to one CUDA context's copy of this
// module, so it is cached per context, under the context's unique id (an id
// is never reused within a process, unlike a context handle, which a new
// context created after cudaDeviceReset may take over).
typedef CUresult (*CtxGetCurrentFn)(CUcontext *);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long *);

struct CtxFns {
    CtxGetCurrentFn get_current = nullptr;
    CtxGetIdFn get_id = nullptr;
};

const CtxFns &ctx_fns() {
    static CtxFns fns;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fns.get_current = reinterpret_cast<CtxGetCurrentFn>(p);
        p = nullptr;
        if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fns.get_id = reinterpret_cast<CtxGetIdFn>(p);
    });
    return fns;
}

constexpr int kNoAllocCacheSlots = 64;
std::mutex g_noalloc_mutex;
unsigned long long g_noalloc_ctx[kNoAllocCacheSlots] = {};   // context ids (0 = free slot)
void *g_noalloc_ptr[kNoAllocCacheSlots] = {};                // the array's address in that context

// Id of the current context, or 0 if there is none yet.
bool current_ctx_id(unsigned long long *id) {
    const CtxFns &f = ctx_fns();
    if (!f.get_current || !f.get_id) return false;
    CUcontext ctx = nullptr;
    if (f.get_current(&ctx) != CUDA_SUCCESS) return false;
    *id = 0;
    return !ctx || f.get_id(ctx, id) == CUDA_SUCCESS;
}

// Resolves the device address of the static array in the current context
// (host code cannot use the symbol's name as a device pointer).  The first
// lookup in a context calls cudaGetSymbolAddress, which also creates the
// device's primary context when no context is current yet.
streamkl_status noalloc_scratch(void **out) {
    unsigned long long id = 0;
    if (!current_ctx_id(&id)) return STREAMKL_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    for (int k = 0; id && k < kNoAllocCacheSlots; ++k)
        if (g_noalloc_ctx[k] == id) {
            *out = g_noalloc_ptr[k];
            return STREAMKL_OK;
        }
    void *ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) return STREAMKL_ERR_CUDA;
    if (!id && !current_ctx_id(&id)) return STREAMKL_ERR_CUDA;
    for (int k = 0; id && k < kNoAllocCacheSlots; ++k)
        if (g_noalloc_ctx[k] == 0) {              // remember it (a full table only means a lookup per call)
            g_noalloc_ctx[k] = id;
            g_noalloc_ptr[k] = ptr;
            break;
        }
    *out = ptr;
    return STREAMKL_OK;
}

}  // namespace

extern "C" streamkl_status streamkl_fwd_noalloc(const void *q_t, const void *k_t, const void *q_s, const void *k_s,
                                                int B, int H, int N_Q, int N_K, int d_t, int d_s, float scale_t,
                                                float scale_s, int causal, float *kl, float *lse_t, float *lse_s,
                                                float *loss_mean, void *stream, unsigned int *status_out) {
    // every problem runs with the minimum workspace (key splitting, which
    // needs more, is only used when the caller's workspace has room for it)
    static_assert(kWorkspaceBytes <= kNoAllocScratchBytes, "the array holds the minimum workspace");
    // Arguments first, with no CUDA call: a rejected call must not clear the
    // status word that an earlier call, maybe still running, may yet set.
    streamkl_status st = check_shape(B, H, N_Q, N_K, d_t, d_s, causal, scale_t, scale_s);
    if (st != STREAMKL_OK) return st;
    if ((st = fwd_check_pointers(q_t, k_t, q_s, k_s, B, H, N_Q, kl, lse_t, lse_s)) != STREAMKL_OK) return st;
    if ((long long)B * H * N_Q > 0 && (st = check_device()) != STREAMKL_OK) return st;
    void *scratch = nullptr;
    if ((st = noalloc_scratch(&scratch)) != STREAMKL_OK) return st;
    cudaStream_t s = (cudaStream_t)stream;
    // the status word must start at zero for this call
    if (cudaMemsetAsync(scratch, 0, kNoAllocScratchBytes, s) != cudaSuccess) return STREAMKL_ERR_CUDA;
    st = streamkl_fwd(q_t, k_t, q_s, k_s, B, H, N_Q, N_K, d_t, d_s, scale_t, scale_s, causal, kl, lse_t, lse_s,
                      loss_mean, scratch, kNoAllocScratchBytes, stream);
    if (st != STREAMKL_OK || !status_out) return st;
    // the caller asked for the device status: wait for this call and read it
    unsigned int word = 0;
    if (cudaMemcpyAsync(&word, scratch, sizeof word, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
        return STREAMKL_ERR_CUDA;
    *status_out = word;
    return (word & kStatusTimeout) ? STREAMKL_ERR_TIMEOUT : STREAMKL_OK;
}
