// fa_api.cu -- the C ABI declared in include/fa.h: argument checks, TMA
// descriptor encoding and kernel launches.  No device memory is allocated here.
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <vector>

#include "fa.h"
#include "fa_bwd.cuh"
#include "fa_bwd_dq.cuh"
#include "fa_bwd_split.cuh"
#include "fa_fwd.cuh"
#include "fa_fwd_fp8.cuh"

namespace {

constexpr float kLog2e = 1.4426950408889634f;

// ---------------------------------------------------------------- profiling
struct ProfRecord {
    int kind;
    cudaEvent_t start, stop;
};
std::mutex g_prof_mu;
bool g_prof_on = false;
std::vector<ProfRecord> g_prof;

// Records events around one kernel launch when profiling is on.
class ProfScope {
   public:
    ProfScope(int kind, cudaStream_t s) : kind_(kind), s_(s) {
        std::lock_guard<std::mutex> g(g_prof_mu);
        if (!g_prof_on) return;
        if (cudaEventCreate(&a_) != cudaSuccess || cudaEventCreate(&b_) != cudaSuccess) return;
        active_ = cudaEventRecord(a_, s_) == cudaSuccess;
    }
    ~ProfScope() {
        if (!active_) return;
        cudaEventRecord(b_, s_);
        std::lock_guard<std::mutex> g(g_prof_mu);
        g_prof.push_back({kind_, a_, b_});
    }

   private:
    int kind_;
    cudaStream_t s_;
    cudaEvent_t a_ = nullptr, b_ = nullptr;
    bool active_ = false;
};

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault,
                                             &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}

// [BH][N][d] 16-bit tensor seen as a 3-D TMA map {d, N, BH} with 64 x rows x 1
// boxes and 128-byte swizzle; rows past N read as zeros.
int make_map(CUtensorMap *map, const void *base, int d, int N, long long BH, int dtype, int box_rows) {
    auto enc = encode_fn();
    if (!enc) return FA_ERR_CUDA;
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N),
                          static_cast<cuuint64_t>(BH)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2,
                             static_cast<cuuint64_t>(N) * static_cast<cuuint64_t>(d) * 2};
    cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(map, dtype == FA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                     3, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? FA_OK : FA_ERR_CUDA;
}

// Packed [total][H][d] 16-bit tensor (variable-length batches) seen as a 3-D
// TMA map {d, total, H}: the same 64 x rows x 1 boxes as make_map, with the
// row coordinate running over the packed rows of one head (stride H * d
// elements) and the plane over heads (stride d).
int make_map_packed(CUtensorMap *map, const void *base, int d, int total, int H, int dtype, int box_rows) {
    auto enc = encode_fn();
    if (!enc) return FA_ERR_CUDA;
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(total), static_cast<cuuint64_t>(H)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(H) * static_cast<cuuint64_t>(d) * 2,
                             static_cast<cuuint64_t>(d) * 2};
    cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(map, dtype == FA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                     3, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? FA_OK : FA_ERR_CUDA;
}

// [BH][N][d] E4M3 codes as a 3-D TMA map {d, N, BH} with d x 128 x 1 boxes
// (d = 128: one 128-byte swizzle atom per row); rows past N read as zeros.
int make_map8(CUtensorMap *map, const void *base, int d, int N, long long BH) {
    auto enc = encode_fn();
    if (!enc) return FA_ERR_CUDA;
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(BH)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(d),
                             static_cast<cuuint64_t>(N) * static_cast<cuuint64_t>(d)};
    // one swizzle atom wide: 128 bytes (d = 256: two boxes per 128-row
    // tile), or 64 bytes with the 64-byte swizzle at d = 64
    cuuint32_t box[3] = {static_cast<cuuint32_t>(d < 128 ? d : 128), 128, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void *>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, d < 128 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? FA_OK : FA_ERR_CUDA;
}

// One attention problem as the entry points describe it.  Window sides and
// ALiBi are optional (negative side = unbounded, null slopes = no bias).
struct Problem {
    int B, H, Nq, Nk, d;
    float scale;
    int causal;
    int win_left, win_right;
    const float *alibi;        // DEVICE [H]
    const uint8_t *mask;       // DEVICE [ceil(Nq/128)][ceil(Nk/128)]
    int dtype;
    long long BH() const { return static_cast<long long>(B) * H; }
    int off() const { return Nk - Nq; }
    int wl() const { return win_left < 0 ? fa::kUnbounded : (win_left < fa::kUnbounded ? win_left : fa::kUnbounded); }
    int wr() const {   // causal caps the right side at the diagonal
        if (causal) return 0;
        return win_right < 0 ? fa::kUnbounded : (win_right < fa::kUnbounded ? win_right : fa::kUnbounded);
    }
    int mode() const { return (causal ? fa::kCausal : 0) | (mask ? fa::kSparse : 0); }
    // square, windowless, unbiased problems run the plain (non-GENERAL) kernels
    bool general() const { return Nq != Nk || win_left >= 0 || win_right >= 0 || alibi != nullptr; }
};

Problem square(int B, int H, int N, int d, float scale, int causal, const uint8_t *mask, int dtype) {
    return Problem{B, H, N, N, d, scale, causal, -1, -1, nullptr, mask, dtype};
}

int check_problem(const Problem &pr) {
    if (pr.B < 1 || pr.H < 1 || pr.Nq < 1 || pr.Nk < 1) return FA_ERR_INVALID_ARG;
    if (pr.Nq > fa::kMaxRows || pr.Nk > fa::kMaxRows) return FA_ERR_UNSUPPORTED;
    if (pr.dtype != FA_F16 && pr.dtype != FA_BF16) return FA_ERR_INVALID_ARG;
    if (!std::isfinite(pr.scale) || !(pr.scale > 0.f)) return FA_ERR_INVALID_ARG;
    if (pr.d != 64 && pr.d != 128 && pr.d != 256) return FA_ERR_UNSUPPORTED;
    if (pr.BH() > 0x7fffffffLL) return FA_ERR_UNSUPPORTED;
    if (pr.alibi && (reinterpret_cast<uintptr_t>(pr.alibi) & 3u)) return FA_ERR_MISALIGNED;
    return FA_OK;
}

template <int D, int NQ, int NSK, int NSV, bool BF16, bool GENERAL, bool VARLEN = false>
int launch_fwd(const CUtensorMap &mq, const CUtensorMap &mk, const CUtensorMap &mv, const CUtensorMap &mo,
               const fa::FwdParams &p, int BH, cudaStream_t stream) {
    using C = fa::FwdCfg<D, NQ, NSK, NSV>;
    auto kern = fa::fwd_kernel<D, NQ, NSK, NSV, BF16, GENERAL, VARLEN>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) != cudaSuccess)
        return FA_ERR_CUDA;
    const long long items = static_cast<long long>(BH) * ((p.nqb + NQ - 1) / NQ);
    if (items > 0x7fffffffLL) return FA_ERR_UNSUPPORTED;
    fa::FwdParams pp = p;
    pp.nitems = static_cast<int>(items);
    // two query tiles per item: one resident CTA per SM runs its share of
    // the items in turn; one tile per item (d = 256): one CTA per item
    long long ctas = items;
    if (NQ == 2) {
        int dev = 0, sms = 0;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1)
            return FA_ERR_CUDA;
        ctas = std::min<long long>(items, sms);
    }
    dim3 grid(static_cast<unsigned>(ctas));
    ProfScope prof(0, stream);
    kern<<<grid, C::kThreads, C::kSmemBytes, stream>>>(mq, mk, mv, mo, pp);
    return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

template <bool BF16, bool GENERAL, bool VARLEN = false>
int dispatch_fwd(int d, const CUtensorMap &mq, const CUtensorMap &mk, const CUtensorMap &mv, const CUtensorMap &mo,
                 const fa::FwdParams &p, int BH, cudaStream_t s) {
    switch (d) {
        case 64: return launch_fwd<64, 2, 6, 4, BF16, GENERAL, VARLEN>(mq, mk, mv, mo, p, BH, s);
        case 128: return launch_fwd<128, 2, 3, 2, BF16, GENERAL, VARLEN>(mq, mk, mv, mo, p, BH, s);
        case 256: return launch_fwd<256, 1, 1, 1, BF16, GENERAL, VARLEN>(mq, mk, mv, mo, p, BH, s);
        default: return FA_ERR_UNSUPPORTED;
    }
}

int fwd_impl(const void *q, const void *k, const void *v, void *o, float *lse, const Problem &pr, void *stream) {
    if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
    int rc = check_problem(pr);
    if (rc != FA_OK) return rc;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
        return FA_ERR_MISALIGNED;
    const int BH = static_cast<int>(pr.BH());
    if (static_cast<long long>(BH) * ((pr.Nq + 127) / 128) > 0x7fffffffLL) return FA_ERR_UNSUPPORTED;   // 1-D grid
    CUtensorMap mq, mk, mv, mo;
    if ((rc = make_map(&mq, q, pr.d, pr.Nq, BH, pr.dtype, 128)) != FA_OK) return rc;
    if ((rc = make_map(&mo, o, pr.d, pr.Nq, BH, pr.dtype, 128)) != FA_OK) return rc;
    if ((rc = make_map(&mk, k, pr.d, pr.Nk, BH, pr.dtype, 128)) != FA_OK) return rc;
    if ((rc = make_map(&mv, v, pr.d, pr.Nk, BH, pr.dtype, 128)) != FA_OK) return rc;
    fa::FwdParams p{};
    p.lse = lse;
    p.mask = pr.mask;
    p.alibi = pr.alibi;
    p.Nq = pr.Nq;
    p.Nk = pr.Nk;
    p.off = pr.off();
    p.wl = pr.wl();
    p.wr = pr.wr();
    p.nqb = (pr.Nq + 127) / 128;
    p.nkb = (pr.Nk + 127) / 128;
    p.nbh = BH;
    p.H = pr.H;
    p.mode = pr.mode();
    p.scale = pr.scale;
    p.scale_log2 = pr.scale * kLog2e;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const bool general = pr.general();
    if (pr.dtype == FA_BF16)
        return general ? dispatch_fwd<true, true>(pr.d, mq, mk, mv, mo, p, BH, s)
                       : dispatch_fwd<true, false>(pr.d, mq, mk, mv, mo, p, BH, s);
    return general ? dispatch_fwd<false, true>(pr.d, mq, mk, mv, mo, p, BH, s)
                   : dispatch_fwd<false, false>(pr.d, mq, mk, mv, mo, p, BH, s);
}

// A packed variable-length batch: B sequences of at most Nq (Nk) query (key)
// rows, total_q (total_k) packed rows in all, lengths in cu_q / cu_k.
struct Packed {
    const int *cu_q, *cu_k;
    int total_q, total_k;
};

int check_packed(const Packed &pk, const Problem &pr) {
    if (!pk.cu_q || !pk.cu_k) return FA_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(pk.cu_q) & 3u) || (reinterpret_cast<uintptr_t>(pk.cu_k) & 3u))
        return FA_ERR_MISALIGNED;
    if (pk.total_q < 1 || pk.total_k < 1 || pr.Nq > pk.total_q || pr.Nk > pk.total_k) return FA_ERR_INVALID_ARG;
    if (pr.mask) return FA_ERR_UNSUPPORTED;
    if (static_cast<long long>(pk.total_q) * pr.H > 0x7fffffffLL ||
        static_cast<long long>(pk.total_k) * pr.H > 0x7fffffffLL)
        return FA_ERR_UNSUPPORTED;
    return FA_OK;
}

int fwd_varlen_impl(const void *q, const void *k, const void *v, void *o, float *lse, const Problem &pr,
                    const Packed &pk, void *stream) {
    if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
    int rc = check_problem(pr);
    if (rc != FA_OK) return rc;
    if ((rc = check_packed(pk, pr)) != FA_OK) return rc;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
        return FA_ERR_MISALIGNED;
    const int BH = static_cast<int>(pr.BH());
    if (static_cast<long long>(BH) * ((pr.Nq + 127) / 128) > 0x7fffffffLL) return FA_ERR_UNSUPPORTED;
    CUtensorMap mq, mk, mv, mo;
    if ((rc = make_map_packed(&mq, q, pr.d, pk.total_q, pr.H, pr.dtype, 128)) != FA_OK) return rc;
    if ((rc = make_map_packed(&mo, o, pr.d, pk.total_q, pr.H, pr.dtype, 128)) != FA_OK) return rc;
    if ((rc = make_map_packed(&mk, k, pr.d, pk.total_k, pr.H, pr.dtype, 128)) != FA_OK) return rc;
    if ((rc = make_map_packed(&mv, v, pr.d, pk.total_k, pr.H, pr.dtype, 128)) != FA_OK) return rc;
    fa::FwdParams p{};
    p.lse = lse;
    p.mask = nullptr;
    p.alibi = pr.alibi;
    p.Nq = pr.Nq;   // the longest sequences: they size the item grid
    p.Nk = pr.Nk;
    p.off = pr.off();
    p.wl = pr.wl();
    p.wr = pr.wr();
    p.nqb = (pr.Nq + 127) / 128;
    p.nkb = (pr.Nk + 127) / 128;
    p.nbh = BH;
    p.H = pr.H;
    p.mode = pr.mode();
    p.scale = pr.scale;
    p.scale_log2 = pr.scale * kLog2e;
    p.cu_q = pk.cu_q;
    p.cu_k = pk.cu_k;
    p.o = o;
    p.total_q = pk.total_q;
    p.total_k = pk.total_k;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (pr.dtype == FA_BF16) return dispatch_fwd<true, true, true>(pr.d, mq, mk, mv, mo, p, BH, s);
    return dispatch_fwd<false, true, true>(pr.d, mq, mk, mv, mo, p, BH, s);
}


// D = rowsum(dO o O), LSE * log2(e) (padded rows: +inf) and dQacc = 0.
template <int D, bool BF16>
int launch_bwd_pre(const void *o, const void *dout, const float *lse, float *lse2, float *dvec, float *dqacc,
                   int BH, int N, int Npad, cudaStream_t stream) {
    constexpr int TPR = D / 8;
    const long long threads = static_cast<long long>(BH) * Npad * TPR;
    const unsigned blocks = static_cast<unsigned>((threads + 255) / 256);
    ProfScope prof(1, stream);
    fa::bwd_pre_kernel<D, BF16><<<blocks, 256, 0, stream>>>(
        static_cast<const uint4 *>(o), static_cast<const uint4 *>(dout), lse, lse2, dvec,
        reinterpret_cast<float4 *>(dqacc), N, Npad, BH);
    return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

// dQ = scale * dQacc in the 16-bit type.
template <bool BF16>
int launch_bwd_post(const float *dqacc, void *dq, long long elems, float scale, cudaStream_t stream) {
    const long long n8 = elems / 8;
    const unsigned blocks = static_cast<unsigned>((n8 + 255) / 256);
    ProfScope prof(3, stream);
    fa::bwd_post_kernel<BF16><<<blocks, 256, 0, stream>>>(reinterpret_cast<const float4 *>(dqacc),
                                                           static_cast<uint4 *>(dq), scale, n8);
    return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

struct BwdBuffers {
    const void *q, *k, *v, *o, *dout;
    const float *lse;
    void *dq, *dk, *dv, *workspace;
};

// The deterministic dQ pass: one CTA per 128-row query tile (fa_bwd_dq.cuh).
template <int D, bool BF16, bool GENERAL>
int launch_bwd_dq(const BwdBuffers &bb, const Problem &pr, fa::BwdParams p, const CUtensorMap &mk,
                  const CUtensorMap &mv, cudaStream_t stream) {
    using C = fa::DqCfg<D>;
    const int BH = static_cast<int>(pr.BH());
    CUtensorMap mq, mdo;
    int rc;
    if ((rc = make_map(&mq, bb.q, D, pr.Nq, BH, pr.dtype, 128)) != FA_OK) return rc;
    if ((rc = make_map(&mdo, bb.dout, D, pr.Nq, BH, pr.dtype, 128)) != FA_OK) return rc;
    CUtensorMap mdq;
    if ((rc = make_map(&mdq, bb.dq, D, pr.Nq, BH, pr.dtype, 128)) != FA_OK) return rc;
    p.nqt = (pr.Nq + 127) / 128;
    p.dq = bb.dq;
    auto kern = fa::bwd_dq_kernel<D, BF16, GENERAL>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) != cudaSuccess)
        return FA_ERR_CUDA;
    const dim3 grid(static_cast<unsigned>(static_cast<long long>(BH) * p.nqt));
    ProfScope prof(4, stream);
    kern<<<grid, C::kThreads, C::kSmemBytes, stream>>>(mq, mk, mv, mdo, mdq, p);
    return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

// Three launches: pre-pass, main kernel (Kernel: a bwd_kernel or bwd_split_kernel
// instantiation, BM query rows per tile, `split` CTAs per key block), then the
// post-pass -- or, deterministic, the main kernel without dQ and the dQ pass.
template <int D, int BM, bool BF16, bool GENERAL, typename Kernel>
int launch_bwd(Kernel kern, int smem_bytes, int threads, int split, const BwdBuffers &bb, const Problem &pr,
               bool deterministic, cudaStream_t stream) {
    const int BH = static_cast<int>(pr.BH());
    const int Npad = fa::bwd_npad(pr.Nq);
    float *lse2 = static_cast<float *>(bb.workspace);
    float *dvec = lse2 + static_cast<size_t>(BH) * Npad;
    float *dqacc = deterministic ? nullptr : dvec + static_cast<size_t>(BH) * Npad;
    int rc = launch_bwd_pre<D, BF16>(bb.o, bb.dout, bb.lse, lse2, dvec, dqacc, BH, pr.Nq, Npad, stream);
    if (rc != FA_OK) return rc;
    CUtensorMap mk, mv, mq, mdo, mdk, mdv;
    if ((rc = make_map(&mk, bb.k, D, pr.Nk, BH, pr.dtype, 128)) != FA_OK) return rc;
    if ((rc = make_map(&mdk, bb.dk, D, pr.Nk, BH, pr.dtype, 128)) != FA_OK) return rc;
    if ((rc = make_map(&mdv, bb.dv, D, pr.Nk, BH, pr.dtype, 128)) != FA_OK) return rc;
    if ((rc = make_map(&mv, bb.v, D, pr.Nk, BH, pr.dtype, 128)) != FA_OK) return rc;
    if ((rc = make_map(&mq, bb.q, D, pr.Nq, BH, pr.dtype, BM)) != FA_OK) return rc;
    if ((rc = make_map(&mdo, bb.dout, D, pr.Nq, BH, pr.dtype, BM)) != FA_OK) return rc;
    fa::BwdParams p;
    p.lse2 = lse2;
    p.dvec = dvec;
    p.dqacc = dqacc;
    p.dq = nullptr;
    p.dk = bb.dk;
    p.dv = bb.dv;
    p.mask = pr.mask;
    p.alibi = pr.alibi;
    p.Nq = pr.Nq;
    p.Nk = pr.Nk;
    p.off = pr.off();
    p.wl = pr.wl();
    p.wr = pr.wr();
    p.H = pr.H;
    p.Npad = Npad;
    p.nkb = (pr.Nk + 127) / 128;
    p.nqt = (pr.Nq + BM - 1) / BM;
    p.nbh = BH;
    p.mode = pr.mode();
    p.scale = pr.scale;
    p.scale_log2 = pr.scale * kLog2e;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes) != cudaSuccess)
        return FA_ERR_CUDA;
    {
        // one-dimensional grid of BH x key blocks (x split) CTAs
        const dim3 grid(static_cast<unsigned>(static_cast<long long>(BH) * p.nkb * split));
        ProfScope prof(2, stream);
        kern<<<grid, threads, smem_bytes, stream>>>(mk, mv, mq, mdo, mdk, mdv, p);
    }
    if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
    if (deterministic) return launch_bwd_dq<D, BF16, GENERAL>(bb, pr, p, mk, mv, stream);
    return launch_bwd_post<BF16>(dqacc, bb.dq, static_cast<long long>(BH) * pr.Nq * D, pr.scale, stream);
}

template <bool BF16, bool GENERAL>
int dispatch_bwd(const BwdBuffers &bb, const Problem &pr, bool det, cudaStream_t s) {
    switch (pr.d) {
        case 64: {
            using C = fa::BwdCfg<64, 3>;
            return launch_bwd<64, 128, BF16, GENERAL>(fa::bwd_kernel<64, 3, BF16, GENERAL>, C::kSmemBytes,
                                                      C::kThreads, 1, bb, pr, det, s);
        }
        case 128: {
            using C = fa::BwdCfg<128, 2>;
            return launch_bwd<128, 128, BF16, GENERAL>(fa::bwd_kernel<128, 2, BF16, GENERAL>, C::kSmemBytes,
                                                       C::kThreads, 1, bb, pr, det, s);
        }
        case 256: {
            using C = fa::BwdSplitCfg<256, 64, 2, 1, 2, true>;
            return launch_bwd<256, 64, BF16, GENERAL>(fa::bwd_split_kernel<256, 64, 2, 1, 2, true, BF16, GENERAL>,
                                                      C::kSmemBytes, C::kThreads, 2, bb, pr, det, s);
        }
        default: return FA_ERR_UNSUPPORTED;
    }
}

// Workspace of the deterministic backward: LSE * log2(e) and D only (no fp32
// dQ accumulator).
size_t bwd_det_workspace_bytes(long long BH, int Nq) { return 2 * static_cast<size_t>(BH) * fa::bwd_npad(Nq) * 4; }

int bwd_impl(const BwdBuffers &bb, size_t workspace_bytes, const Problem &pr, void *stream,
             bool deterministic = false) {
    if (!bb.q || !bb.k || !bb.v || !bb.o || !bb.dout || !bb.lse || !bb.dq || !bb.dk || !bb.dv)
        return FA_ERR_INVALID_ARG;
    int rc = check_problem(pr);
    if (rc != FA_OK) return rc;
    const void *ptrs[] = {bb.q, bb.k, bb.v, bb.o, bb.dout, bb.lse, bb.dq, bb.dk, bb.dv};
    for (const void *ptr : ptrs)
        if (!aligned16(ptr)) return FA_ERR_MISALIGNED;
    if (pr.BH() * (2LL * ((pr.Nk + 127) / 128)) > 0x7fffffffLL) return FA_ERR_UNSUPPORTED;   // one-dimensional grids
    if (pr.BH() * ((pr.Nq + 127LL) / 128) > 0x7fffffffLL) return FA_ERR_UNSUPPORTED;
    const size_t need = deterministic ? bwd_det_workspace_bytes(pr.BH(), pr.Nq)
                                      : fa::bwd_workspace_bytes(pr.BH(), pr.Nq, pr.d);
    if (!bb.workspace || workspace_bytes < need) return FA_ERR_WORKSPACE;
    if (!aligned16(bb.workspace)) return FA_ERR_MISALIGNED;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const bool general = pr.general();
    const bool det = deterministic;
    if (pr.dtype == FA_BF16)
        return general ? dispatch_bwd<true, true>(bb, pr, det, s) : dispatch_bwd<true, false>(bb, pr, det, s);
    return general ? dispatch_bwd<false, true>(bb, pr, det, s) : dispatch_bwd<false, false>(bb, pr, det, s);
}

// ---------------------------------------------------------------- packed batches
// Workspace of the packed backward: lse2 and D [BH][Npad] (Npad = the longest
// query sequence rounded up to 128), then (not in the deterministic form) the
// fp32 dQ accumulator [H][total_q][d].
size_t bwd_varlen_workspace_bytes(long long BH, int H, int total_q, int max_nq, int d, bool deterministic) {
    return 2 * static_cast<size_t>(BH) * fa::bwd_npad(max_nq) * 4 +
           (deterministic ? 0 : static_cast<size_t>(H) * static_cast<size_t>(total_q) * d * 4);
}

// The packed backward: pre-pass, key-block kernel (bwd_kernel at d <= 128,
// bwd_split_kernel at d = 256; BM-row query tiles), then the post-pass -- or,
// deterministic, the key-block kernel without dQ and the dQ pass.
template <int D, int BM, bool BF16, typename Kernel>
int launch_bwd_varlen(Kernel kern, int smem_bytes, int threads, int split, const BwdBuffers &bb, const Problem &pr,
                      const Packed &pk, bool deterministic, cudaStream_t stream) {
    const int BH = static_cast<int>(pr.BH());
    const int Npad = fa::bwd_npad(pr.Nq);
    float *lse2 = static_cast<float *>(bb.workspace);
    float *dvec = lse2 + static_cast<size_t>(BH) * Npad;
    float *dqacc = deterministic ? nullptr : dvec + static_cast<size_t>(BH) * Npad;
    {
        constexpr int TPR = D / 8;
        const long long nthreads = static_cast<long long>(BH) * Npad * TPR;
        const unsigned blocks = static_cast<unsigned>((nthreads + 255) / 256);
        ProfScope prof(1, stream);
        fa::bwd_pre_varlen_kernel<D, BF16><<<blocks, 256, 0, stream>>>(
            static_cast<const uint4 *>(bb.o), static_cast<const uint4 *>(bb.dout), bb.lse, lse2, dvec,
            reinterpret_cast<float4 *>(dqacc), pk.cu_q, pr.H, pk.total_q, pr.Nq, Npad, BH);
        if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
    }
    CUtensorMap mk, mv, mq, mdo, mdk, mdv;
    int rc;
    if ((rc = make_map_packed(&mk, bb.k, D, pk.total_k, pr.H, pr.dtype, 128)) != FA_OK) return rc;
    if ((rc = make_map_packed(&mdk, bb.dk, D, pk.total_k, pr.H, pr.dtype, 128)) != FA_OK) return rc;
    if ((rc = make_map_packed(&mdv, bb.dv, D, pk.total_k, pr.H, pr.dtype, 128)) != FA_OK) return rc;
    if ((rc = make_map_packed(&mv, bb.v, D, pk.total_k, pr.H, pr.dtype, 128)) != FA_OK) return rc;
    if ((rc = make_map_packed(&mq, bb.q, D, pk.total_q, pr.H, pr.dtype, BM)) != FA_OK) return rc;
    if ((rc = make_map_packed(&mdo, bb.dout, D, pk.total_q, pr.H, pr.dtype, BM)) != FA_OK) return rc;
    fa::BwdParams p{};
    p.lse2 = lse2;
    p.dvec = dvec;
    p.dqacc = dqacc;
    p.dq = nullptr;
    p.dk = bb.dk;
    p.dv = bb.dv;
    p.mask = nullptr;
    p.alibi = pr.alibi;
    p.Nq = pr.Nq;   // the longest sequences
    p.Nk = pr.Nk;
    p.off = pr.off();
    p.wl = pr.wl();
    p.wr = pr.wr();
    p.H = pr.H;
    p.Npad = Npad;
    p.nkb = (pr.Nk + 127) / 128;
    p.nqt = (pr.Nq + BM - 1) / BM;
    p.nbh = BH;
    p.mode = pr.mode();
    p.scale = pr.scale;
    p.scale_log2 = pr.scale * kLog2e;
    p.cu_q = pk.cu_q;
    p.cu_k = pk.cu_k;
    p.total_q = pk.total_q;
    p.total_k = pk.total_k;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes) != cudaSuccess)
        return FA_ERR_CUDA;
    {
        // B x (key blocks of the longest sequence) x H (x split), sequence
        // major; CTAs past their own sequence's keys return at once
        const dim3 grid(static_cast<unsigned>(static_cast<long long>(BH) * p.nkb * split));
        ProfScope prof(2, stream);
        kern<<<grid, threads, smem_bytes, stream>>>(mk, mv, mq, mdo, mdk, mdv, p);
        if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
    }
    if (deterministic) {
        using C = fa::DqCfg<D>;
        CUtensorMap mq1, mdo1, mdq;
        if ((rc = make_map_packed(&mq1, bb.q, D, pk.total_q, pr.H, pr.dtype, 128)) != FA_OK) return rc;
        if ((rc = make_map_packed(&mdo1, bb.dout, D, pk.total_q, pr.H, pr.dtype, 128)) != FA_OK) return rc;
        if ((rc = make_map_packed(&mdq, bb.dq, D, pk.total_q, pr.H, pr.dtype, 128)) != FA_OK) return rc;
        p.nqt = (pr.Nq + 127) / 128;
        p.dq = bb.dq;
        auto dkern = fa::bwd_dq_kernel<D, BF16, true, true>;
        if (cudaFuncSetAttribute(dkern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) != cudaSuccess)
            return FA_ERR_CUDA;
        // B x (query tiles of the longest sequence) x H, sequence major
        const dim3 grid(static_cast<unsigned>(static_cast<long long>(BH) * p.nqt));
        ProfScope prof(4, stream);
        dkern<<<grid, C::kThreads, C::kSmemBytes, stream>>>(mq1, mk, mv, mdo1, mdq, p);
        return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
    }
    {
        const long long n8 = static_cast<long long>(pr.H) * pk.total_q * (D / 8);
        const unsigned blocks = static_cast<unsigned>((n8 + 255) / 256);
        ProfScope prof(3, stream);
        fa::bwd_post_varlen_kernel<D, BF16><<<blocks, 256, 0, stream>>>(reinterpret_cast<const float4 *>(dqacc),
                                                                         static_cast<uint4 *>(bb.dq), pr.scale,
                                                                         pr.H, pk.total_q);
    }
    return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

template <bool BF16>
int dispatch_bwd_varlen(const BwdBuffers &bb, const Problem &pr, const Packed &pk, bool det, cudaStream_t s) {
    switch (pr.d) {
        case 64: {
            using C = fa::BwdCfg<64, 3>;
            return launch_bwd_varlen<64, 128, BF16>(fa::bwd_kernel<64, 3, BF16, true, true>, C::kSmemBytes,
                                                    C::kThreads, 1, bb, pr, pk, det, s);
        }
        case 128: {
            using C = fa::BwdCfg<128, 2>;
            return launch_bwd_varlen<128, 128, BF16>(fa::bwd_kernel<128, 2, BF16, true, true>, C::kSmemBytes,
                                                     C::kThreads, 1, bb, pr, pk, det, s);
        }
        case 256: {
            using C = fa::BwdSplitCfg<256, 64, 2, 1, 2, true>;
            return launch_bwd_varlen<256, 64, BF16>(fa::bwd_split_kernel<256, 64, 2, 1, 2, true, BF16, true, true>,
                                                    C::kSmemBytes, C::kThreads, 2, bb, pr, pk, det, s);
        }
        default: return FA_ERR_UNSUPPORTED;
    }
}

int bwd_varlen_impl(const BwdBuffers &bb, size_t workspace_bytes, const Problem &pr, const Packed &pk,
                    void *stream, bool deterministic) {
    if (!bb.q || !bb.k || !bb.v || !bb.o || !bb.dout || !bb.lse || !bb.dq || !bb.dk || !bb.dv)
        return FA_ERR_INVALID_ARG;
    int rc = check_problem(pr);
    if (rc != FA_OK) return rc;
    if ((rc = check_packed(pk, pr)) != FA_OK) return rc;
    const void *ptrs[] = {bb.q, bb.k, bb.v, bb.o, bb.dout, bb.lse, bb.dq, bb.dk, bb.dv};
    for (const void *ptr : ptrs)
        if (!aligned16(ptr)) return FA_ERR_MISALIGNED;
    if (pr.BH() * 2LL * ((pr.Nk + 127LL) / 128) > 0x7fffffffLL) return FA_ERR_UNSUPPORTED;   // one-dimensional grids
    if (pr.BH() * ((pr.Nq + 127LL) / 128) > 0x7fffffffLL) return FA_ERR_UNSUPPORTED;
    if (pr.BH() * fa::bwd_npad(pr.Nq) * (pr.d / 8) > 0x7fffffffLL * 256LL) return FA_ERR_UNSUPPORTED;
    const size_t need = bwd_varlen_workspace_bytes(pr.BH(), pr.H, pk.total_q, pr.Nq, pr.d, deterministic);
    if (!bb.workspace || workspace_bytes < need) return FA_ERR_WORKSPACE;
    if (!aligned16(bb.workspace)) return FA_ERR_MISALIGNED;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (pr.dtype == FA_BF16) return dispatch_bwd_varlen<true>(bb, pr, pk, deterministic, s);
    return dispatch_bwd_varlen<false>(bb, pr, pk, deterministic, s);
}

// ---------------------------------------------------------------- fa_bwd_noalloc
// Scratch for fa_bwd_noalloc, resident on every device that loads the library.
// Host code must not use this name as a pointer: on the host it is only a
// stand-in for the symbol, so the device address is looked up per device.
static __device__ __align__(256) unsigned char g_noalloc_scratch[FA_NOALLOC_SCRATCH_BYTES];

// The current device's address of g_noalloc_scratch.  Looked up on every
// call (a host-side table lookup once the module is loaded on the device), so
// that no address outlives the context it belongs to: after a
// cudaDeviceReset the module is loaded again and the array may move.
int noalloc_scratch(void **out) {
    void *ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) return FA_ERR_CUDA;
    *out = ptr;
    return FA_OK;
}

// ---------------------------------------------------------------- FP8
template <int D, bool BF16>
int launch_quant(const fa::QuantParams &qp, long long BH, cudaStream_t s) {
    using C = fa::QuantCfg<D>;
    const long long ctas = BH * qp.nb;
    if (ctas > 0x7fffffffLL) return FA_ERR_UNSUPPORTED;
    {
        ProfScope prof(5, s);
        fa::fp8_quant_kernel<D, BF16><<<dim3(static_cast<unsigned>(ctas), 3), C::kThreads, 0, s>>>(qp, 0);
        if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
    }
    {
        ProfScope prof(5, s);
        fa::fp8_quant_kernel<D, BF16><<<dim3(static_cast<unsigned>(ctas), 1), C::kThreads, 0, s>>>(qp, 1);
        if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
    }
    {
        ProfScope prof(5, s);
        fa::fp8_vscale_kernel<<<static_cast<unsigned>((BH + 255) / 256), 256, 0, s>>>(qp.scales[2], qp.nb, BH);
        if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
    }
    return FA_OK;
}

// The FP8 forward: one CTA per NQ query tiles of one (b, h), heaviest first under causal.
template <int D, bool BF16>
int launch_fwd8(const CUtensorMap &mq, const CUtensorMap &mk, const CUtensorMap &mv, const CUtensorMap &mo,
                const fa::Fwd8Params &p, long long BH, cudaStream_t s) {
    using C = fa::Fwd8Cfg<D>;
    auto kern = fa::fwd8_kernel<D, BF16>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes) != cudaSuccess)
        return FA_ERR_CUDA;
    const dim3 grid(static_cast<unsigned>(BH * ((p.nb + C::NQ - 1) / C::NQ)));
    ProfScope prof(6, s);
    kern<<<grid, C::kThreads, C::kSmemBytes, s>>>(mq, mk, mv, mo, p);
    return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

}  // namespace

extern "C" {

FA_API int fa_fp8_quantize_qkv(const void *q, const void *k, const void *v, uint8_t *q8, uint8_t *k8, uint8_t *v8,
                               float *sq, float *sk, float *sv, int B, int H, int N, int d, const float *signs,
                               int dtype, void *stream) {
    if (!q || !k || !v || !q8 || !k8 || !v8 || !sq || !sk || !sv) return FA_ERR_INVALID_ARG;
    if (B < 1 || H < 1 || N < 1) return FA_ERR_INVALID_ARG;
    if (dtype != FA_F16 && dtype != FA_BF16) return FA_ERR_INVALID_ARG;
    if (d != 64 && d != 128 && d != 256) return FA_ERR_UNSUPPORTED;
    const long long BH = static_cast<long long>(B) * H;
    if (BH > 0x7fffffffLL || N > fa::kMaxRows) return FA_ERR_UNSUPPORTED;
    const void *ptrs[] = {q, k, v, q8, k8, v8};
    for (const void *ptr : ptrs)
        if (!aligned16(ptr)) return FA_ERR_MISALIGNED;
    const void *fptrs[] = {sq, sk, sv, signs};
    for (const void *ptr : fptrs)
        if (reinterpret_cast<uintptr_t>(ptr) & 3u) return FA_ERR_MISALIGNED;
    fa::QuantParams qp;
    qp.src[0] = q;
    qp.src[1] = k;
    qp.src[2] = v;
    qp.dst[0] = q8;
    qp.dst[1] = k8;
    qp.dst[2] = v8;
    qp.scales[0] = sq;
    qp.scales[1] = sk;
    qp.scales[2] = sv;
    qp.signs = signs;
    qp.rnorm = static_cast<float>(1.0 / std::sqrt(static_cast<double>(d)));
    qp.N = N;
    qp.nb = (N + 127) / 128;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const bool bf = dtype == FA_BF16;
    switch (d) {
        case 64: return bf ? launch_quant<64, true>(qp, BH, s) : launch_quant<64, false>(qp, BH, s);
        case 128: return bf ? launch_quant<128, true>(qp, BH, s) : launch_quant<128, false>(qp, BH, s);
        default: return bf ? launch_quant<256, true>(qp, BH, s) : launch_quant<256, false>(qp, BH, s);
    }
}

FA_API int fa_fwd_fp8(const uint8_t *q8, const uint8_t *k8, const uint8_t *v8, const float *sq, const float *sk,
                      const float *sv, void *o, float *lse, int B, int H, int N, int d, float scale, int causal,
                      int out_dtype, void *stream) {
    if (!q8 || !k8 || !v8 || !sq || !sk || !sv || !o || !lse) return FA_ERR_INVALID_ARG;
    if (B < 1 || H < 1 || N < 1) return FA_ERR_INVALID_ARG;
    if (out_dtype != FA_F16 && out_dtype != FA_BF16) return FA_ERR_INVALID_ARG;
    if (!std::isfinite(scale) || !(scale > 0.f)) return FA_ERR_INVALID_ARG;
    if (d != 64 && d != 128 && d != 256) return FA_ERR_UNSUPPORTED;
    const long long BH = static_cast<long long>(B) * H;
    if (N > fa::kMaxRows || BH * ((N + 127) / 128) > 0x7fffffffLL) return FA_ERR_UNSUPPORTED;
    const void *ptrs[] = {q8, k8, v8, o, lse};
    for (const void *ptr : ptrs)
        if (!aligned16(ptr)) return FA_ERR_MISALIGNED;
    const void *fptrs[] = {sq, sk, sv};
    for (const void *ptr : fptrs)
        if (reinterpret_cast<uintptr_t>(ptr) & 3u) return FA_ERR_MISALIGNED;
    CUtensorMap mq, mk, mv, mo;
    int rc;
    if ((rc = make_map8(&mq, q8, d, N, BH)) != FA_OK) return rc;
    if ((rc = make_map8(&mk, k8, d, N, BH)) != FA_OK) return rc;
    if ((rc = make_map8(&mv, v8, d, N, BH)) != FA_OK) return rc;
    if ((rc = make_map(&mo, o, d, N, BH, out_dtype, 128)) != FA_OK) return rc;
    fa::Fwd8Params p;
    p.lse = lse;
    p.sq = sq;
    p.sk = sk;
    p.sv = sv;
    p.N = N;
    p.nb = (N + 127) / 128;
    p.nbh = static_cast<int>(BH);
    p.causal = causal ? 1 : 0;
    p.scale_log2 = scale * kLog2e;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (d == 64)
        return out_dtype == FA_BF16 ? launch_fwd8<64, true>(mq, mk, mv, mo, p, BH, s)
                                    : launch_fwd8<64, false>(mq, mk, mv, mo, p, BH, s);
    if (d == 128)
        return out_dtype == FA_BF16 ? launch_fwd8<128, true>(mq, mk, mv, mo, p, BH, s)
                                    : launch_fwd8<128, false>(mq, mk, mv, mo, p, BH, s);
    return out_dtype == FA_BF16 ? launch_fwd8<256, true>(mq, mk, mv, mo, p, BH, s)
                                : launch_fwd8<256, false>(mq, mk, mv, mo, p, BH, s);
}

FA_API int fa_fwd(const void *q, const void *k, const void *v, void *o, float *lse, int B, int H, int N, int d,
                  float scale, int causal, int dtype, void *stream) {
    return fwd_impl(q, k, v, o, lse, square(B, H, N, d, scale, causal, nullptr, dtype), stream);
}

FA_API int fa_fwd_blocksparse(const void *q, const void *k, const void *v, void *o, float *lse,
                              const uint8_t *block_mask, int B, int H, int N, int d, float scale, int causal,
                              int dtype, void *stream) {
    if (!block_mask) return FA_ERR_INVALID_ARG;
    return fwd_impl(q, k, v, o, lse, square(B, H, N, d, scale, causal, block_mask, dtype), stream);
}

FA_API int fa_fwd_ex(const void *q, const void *k, const void *v, void *o, float *lse, int B, int H, int Nq,
                     int Nk, int d, float scale, int causal, int window_left, int window_right,
                     const float *alibi_slopes, const uint8_t *block_mask, int dtype, void *stream) {
    const Problem pr{B, H, Nq, Nk, d, scale, causal, window_left, window_right, alibi_slopes, block_mask, dtype};
    return fwd_impl(q, k, v, o, lse, pr, stream);
}

FA_API int fa_fwd_varlen(const void *q, const void *k, const void *v, void *o, float *lse,
                         const int *cu_seqlens_q, const int *cu_seqlens_k, int B, int H, int total_q, int total_k,
                         int max_seqlen_q, int max_seqlen_k, int d, float scale, int causal, int window_left,
                         int window_right, const float *alibi_slopes, int dtype, void *stream) {
    const Problem pr{B, H, max_seqlen_q, max_seqlen_k, d, scale, causal, window_left, window_right, alibi_slopes,
                     nullptr, dtype};
    const Packed pk{cu_seqlens_q, cu_seqlens_k, total_q, total_k};
    return fwd_varlen_impl(q, k, v, o, lse, pr, pk, stream);
}

FA_API size_t fa_bwd_varlen_workspace_bytes(int B, int H, int total_q, int max_seqlen_q, int d) {
    if (B < 1 || H < 1 || total_q < 1 || max_seqlen_q < 1 || max_seqlen_q > total_q ||
        (d != 64 && d != 128 && d != 256))
        return 0;
    return bwd_varlen_workspace_bytes(static_cast<long long>(B) * H, H, total_q, max_seqlen_q, d, false);
}

FA_API size_t fa_bwd_varlen_deterministic_workspace_bytes(int B, int H, int total_q, int max_seqlen_q, int d) {
    if (fa_bwd_varlen_workspace_bytes(B, H, total_q, max_seqlen_q, d) == 0) return 0;
    return bwd_varlen_workspace_bytes(static_cast<long long>(B) * H, H, total_q, max_seqlen_q, d, true);
}

FA_API int fa_bwd_varlen(const void *q, const void *k, const void *v, const void *o, const void *dout,
                         const float *lse, void *dq, void *dk, void *dv, void *workspace, size_t workspace_bytes,
                         const int *cu_seqlens_q, const int *cu_seqlens_k, int B, int H, int total_q, int total_k,
                         int max_seqlen_q, int max_seqlen_k, int d, float scale, int causal, int window_left,
                         int window_right, const float *alibi_slopes, int dtype, void *stream) {
    const Problem pr{B, H, max_seqlen_q, max_seqlen_k, d, scale, causal, window_left, window_right, alibi_slopes,
                     nullptr, dtype};
    const Packed pk{cu_seqlens_q, cu_seqlens_k, total_q, total_k};
    const BwdBuffers bb{q, k, v, o, dout, lse, dq, dk, dv, workspace};
    return bwd_varlen_impl(bb, workspace_bytes, pr, pk, stream, false);
}

FA_API int fa_bwd_varlen_deterministic(const void *q, const void *k, const void *v, const void *o,
                                       const void *dout, const float *lse, void *dq, void *dk, void *dv,
                                       void *workspace, size_t workspace_bytes, const int *cu_seqlens_q,
                                       const int *cu_seqlens_k, int B, int H, int total_q, int total_k,
                                       int max_seqlen_q, int max_seqlen_k, int d, float scale, int causal,
                                       int window_left, int window_right, const float *alibi_slopes, int dtype,
                                       void *stream) {
    const Problem pr{B, H, max_seqlen_q, max_seqlen_k, d, scale, causal, window_left, window_right, alibi_slopes,
                     nullptr, dtype};
    const Packed pk{cu_seqlens_q, cu_seqlens_k, total_q, total_k};
    const BwdBuffers bb{q, k, v, o, dout, lse, dq, dk, dv, workspace};
    return bwd_varlen_impl(bb, workspace_bytes, pr, pk, stream, true);
}

FA_API size_t fa_bwd_workspace_bytes(int B, int H, int N, int d) {
    if (B < 1 || H < 1 || N < 1 || (d != 64 && d != 128 && d != 256)) return 0;
    return fa::bwd_workspace_bytes(static_cast<long long>(B) * H, N, d);
}

FA_API size_t fa_bwd_ex_workspace_bytes(int B, int H, int Nq, int Nk, int d) {
    if (Nk < 1) return 0;
    return fa_bwd_workspace_bytes(B, H, Nq, d);
}

FA_API int fa_bwd(const void *q, const void *k, const void *v, const void *o, const void *dout, const float *lse,
                  void *dq, void *dk, void *dv, void *workspace, size_t workspace_bytes, int B, int H, int N,
                  int d, float scale, int causal, int dtype, void *stream) {
    const BwdBuffers bb{q, k, v, o, dout, lse, dq, dk, dv, workspace};
    return bwd_impl(bb, workspace_bytes, square(B, H, N, d, scale, causal, nullptr, dtype), stream);
}

FA_API int fa_bwd_blocksparse(const void *q, const void *k, const void *v, const void *o, const void *dout,
                              const float *lse, void *dq, void *dk, void *dv, void *workspace,
                              size_t workspace_bytes, const uint8_t *block_mask, int B, int H, int N, int d,
                              float scale, int causal, int dtype, void *stream) {
    if (!block_mask) return FA_ERR_INVALID_ARG;
    const BwdBuffers bb{q, k, v, o, dout, lse, dq, dk, dv, workspace};
    return bwd_impl(bb, workspace_bytes, square(B, H, N, d, scale, causal, block_mask, dtype), stream);
}

FA_API int fa_bwd_ex(const void *q, const void *k, const void *v, const void *o, const void *dout,
                     const float *lse, void *dq, void *dk, void *dv, void *workspace, size_t workspace_bytes,
                     int B, int H, int Nq, int Nk, int d, float scale, int causal, int window_left,
                     int window_right, const float *alibi_slopes, const uint8_t *block_mask, int dtype,
                     void *stream) {
    const BwdBuffers bb{q, k, v, o, dout, lse, dq, dk, dv, workspace};
    const Problem pr{B, H, Nq, Nk, d, scale, causal, window_left, window_right, alibi_slopes, block_mask, dtype};
    return bwd_impl(bb, workspace_bytes, pr, stream);
}

FA_API size_t fa_bwd_deterministic_workspace_bytes(int B, int H, int Nq, int Nk, int d) {
    if (B < 1 || H < 1 || Nq < 1 || Nk < 1 || (d != 64 && d != 128 && d != 256)) return 0;
    return bwd_det_workspace_bytes(static_cast<long long>(B) * H, Nq);
}

FA_API int fa_bwd_deterministic(const void *q, const void *k, const void *v, const void *o, const void *dout,
                                const float *lse, void *dq, void *dk, void *dv, void *workspace,
                                size_t workspace_bytes, int B, int H, int Nq, int Nk, int d, float scale, int causal,
                                int window_left, int window_right, const float *alibi_slopes,
                                const uint8_t *block_mask, int dtype, void *stream) {
    const BwdBuffers bb{q, k, v, o, dout, lse, dq, dk, dv, workspace};
    const Problem pr{B, H, Nq, Nk, d, scale, causal, window_left, window_right, alibi_slopes, block_mask, dtype};
    return bwd_impl(bb, workspace_bytes, pr, stream, true);
}

FA_API int fa_bwd_noalloc(const void *q, const void *k, const void *v, const void *o, const void *dout,
                          const float *lse, void *dq, void *dk, void *dv, int B, int H, int N, int d, float scale,
                          int causal, int dtype, void *stream) {
    const Problem pr = square(B, H, N, d, scale, causal, nullptr, dtype);
    int rc = check_problem(pr);
    if (rc != FA_OK) return rc;
    const size_t need = fa::bwd_workspace_bytes(pr.BH(), N, d);
    if (need > FA_NOALLOC_SCRATCH_BYTES) return FA_ERR_SCRATCH_LIMIT;
    void *scratch = nullptr;
    if ((rc = noalloc_scratch(&scratch)) != FA_OK) return rc;
    const BwdBuffers bb{q, k, v, o, dout, lse, dq, dk, dv, scratch};
    return bwd_impl(bb, FA_NOALLOC_SCRATCH_BYTES, pr, stream);
}

FA_API const char *fa_status_string(int status) {
    switch (status) {
        case FA_OK: return "ok";
        case FA_ERR_INVALID_ARG: return "invalid argument";
        case FA_ERR_UNSUPPORTED: return "unsupported shape";
        case FA_ERR_MISALIGNED: return "pointer not 16-byte aligned";
        case FA_ERR_WORKSPACE: return "workspace missing or too small";
        case FA_ERR_CUDA: return "CUDA error";
        case FA_ERR_TIMEOUT: return "kernel wait timed out";
        case FA_ERR_SCRATCH_LIMIT: return "problem needs more than the built-in scratch of fa_bwd_noalloc";
        default: return "unknown status";
    }
}

FA_API int fa_last_device_status(void) {
    int v = 0, zero = 0;
    if (cudaDeviceSynchronize() != cudaSuccess) return FA_ERR_CUDA;
    if (cudaMemcpyFromSymbol(&v, fa::g_dev_status, sizeof(int)) != cudaSuccess) return FA_ERR_CUDA;
    if (cudaMemcpyToSymbol(fa::g_dev_status, &zero, sizeof(int)) != cudaSuccess) return FA_ERR_CUDA;
    return v;
}

FA_API int fa_last_timeout_site(int *site) {
    if (!site) return FA_ERR_INVALID_ARG;
    if (cudaDeviceSynchronize() != cudaSuccess) return FA_ERR_CUDA;
    if (cudaMemcpyFromSymbol(site, fa::g_dev_site, 5 * sizeof(int)) != cudaSuccess) return FA_ERR_CUDA;
    return FA_OK;
}

FA_API int fa_profile_enable(int on) {
    std::lock_guard<std::mutex> g(g_prof_mu);
    g_prof_on = on != 0;
    return FA_OK;
}

FA_API int fa_profile_read(float *ms, int *launches) {
    if (!ms || !launches) return FA_ERR_INVALID_ARG;
    std::vector<ProfRecord> recs;
    {
        std::lock_guard<std::mutex> g(g_prof_mu);
        recs.swap(g_prof);
    }
    for (int k = 0; k < FA_PROFILE_KINDS; ++k) {
        ms[k] = 0.f;
        launches[k] = 0;
    }
    int rc = FA_OK;
    for (auto &r : recs) {
        float t = 0.f;
        if (cudaEventSynchronize(r.stop) != cudaSuccess || cudaEventElapsedTime(&t, r.start, r.stop) != cudaSuccess)
            rc = FA_ERR_CUDA;
        ms[r.kind] += t;
        launches[r.kind] += 1;
        cudaEventDestroy(r.start);
        cudaEventDestroy(r.stop);
    }
    return rc;
}

FA_API int fa_version(void) { return 100; }

}  // extern "C"
