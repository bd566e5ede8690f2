// fa_bwd.cuh -- backward kernels of exact attention for sm_100a.
//
// What is computed (per (batch, head); "FlashAttention 深度解析" section 四:
// five matrix products; "FlashAttention原理概览" section 3.2: P is recomputed
// from the saved row statistics instead of being stored):
//   P  = exp(scale * Q K^T - LSE)          (recomputed, never stored)
//   dV = P^T dO,   dP = dO V^T,   D_i = sum_c dO_ic O_ic,
//   dS = P o (dP - D),   dQ = scale * dS K,   dK = scale * dS^T Q.
//
// Three launches on the caller's stream:
//   bwd_pre   D = rowsum(dO o O) into the workspace; zeroes the fp32 dQ accumulator.
//   bwd_main  one CTA per 128-key block (bwd_kernel, d <= 128; the d = 256
//             kernel of fa_bwd_split.cuh splits the block's columns over two
//             CTAs).  The CTA keeps K_j, V_j in shared memory and its dK, dV
//             accumulators in tensor memory while it sweeps the kept 128-row
//             query tiles Q_i, dO_i through an NS-stage TMA ring:
//               S^T  = K_j Q_i^T   and  dP^T = V_j dO_i^T   (tcgen05, TMEM)
//               P^T  (16-bit, written back over S^T in TMEM)
//               dS^T (16-bit swizzled tile in shared memory)
//               dV  += P^T dO_i  (TS form),   dK += dS^T Q_i
//               dQ_i^T = K_j^T dS^T  (M = d), into the dP^T columns once dP^T
//                                   has been read, then fp32 reductions into
//                                   the accumulator by the drain warps.
//   bwd_post  dQ = scale * accumulator, rounded to the 16-bit type.
// The deterministic backward passes a null accumulator: bwd_main then computes
// dK, dV only, and the dQ pass of fa_bwd_dq.cuh replaces the reductions and
// bwd_post.
//
// Warp roles of bwd_kernel (512 threads): warps 0-7 softmax-grad (warp w owns
// TMEM lanes 32 (w mod 4) .. +31, i.e. those keys, for queries
// [64 (w div 4), +64) of the tile) and the dV (warps 0-3) / dK (warps 4-7)
// epilogue; warps 8-11 dQ drain; warp 12 TMA producer (also bulk-copies the
// per-row LSE * log2 e and D of each query tile); warp 13 MMA issuer (owns
// TMEM); warps 14-15 idle.
// TMEM columns: S^T / P^T [0, 128), dP^T [128, 256) (then dQ^T: at d = 128
// every lane is a d index, at d = 64 the M = 64 product puts row m in lane
// 32 (m / 16) + m % 16), dV [256, 256 + d), dK [256 + d, 256 + 2 d).
#pragma once

#include "fa_common.cuh"
#include "fa_fwd.cuh"

namespace fa {

struct BwdParams {
    const float *lse2;    // [BH][Npad] LSE * log2(e) (+inf for rows past Nq or with no visible key)
    const float *dvec;    // [BH][Npad] D = rowsum(dO o O) (0 for rows past Nq)
    float *dqacc;         // [BH][Nq][D] fp32, zeroed by bwd_pre; null: the key-block kernels skip dQ
    void *dq;             // [BH][Nq][D] 16-bit (written by the deterministic dQ pass)
    void *dk;             // [BH][Nk][D] 16-bit
    void *dv;             // [BH][Nk][D] 16-bit
    const uint8_t *mask;  // [ceil(Nq/128)][nkb] block mask (kSparse)
    const float *alibi;   // [H] ALiBi slopes (natural-log units of the score) or null (GENERAL kernels)
    int Nq, Nk;           // query rows and keys per (b, h)
    int off, wl, wr;      // visibility band (see band_any)
    int H;                // heads (head of batch-head bh: bh % H)
    int Npad;             // Nq rounded up to 128: row pitch of lse2 and dvec
    int nkb;              // key blocks (and mask blocks) of 128
    int nqt;              // query tiles of BM rows
    int nbh;              // batch x heads
    int mode;
    float scale;
    float scale_log2;
    // packed variable-length batches (VARLEN kernels): sequence b owns packed
    // rows cu_q[b] .. cu_q[b+1]-1 of q, o, dout, dq and cu_k[b] .. cu_k[b+1]-1
    // of k, v, dk, dv ([rows][H][D]); lse is [H][total_q], lse2 and dvec are
    // [BH][Npad] per (sequence, head) and dqacc is [H][total_q][D].  Nq and
    // Nk above then bound the sequence lengths.
    const int *cu_q;
    const int *cu_k;
    int total_q, total_k;
};

// ---------------------------------------------------------------------------
// bwd_pre: D_i = sum_c dO_ic O_ic, and dQacc = 0
// ---------------------------------------------------------------------------
template <int D, bool BF16>
__global__ void __launch_bounds__(256) bwd_pre_kernel(const uint4 *__restrict__ o, const uint4 *__restrict__ dout,
                                                      const float *__restrict__ lse, float *__restrict__ lse2,
                                                      float *__restrict__ dvec, float4 *__restrict__ dqacc, int N,
                                                      int Npad, long long BH) {
    constexpr int TPR = D / 8;   // threads per row, 8 elements (16 bytes) each
    const long long tid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    const long long prow = tid / TPR;                 // padded row index bh * Npad + n
    const int part = static_cast<int>(tid % TPR);
    const long long bh = prow / Npad;
    const int n = static_cast<int>(prow % Npad);
    const bool valid = bh < BH && n < N;
    const long long row = bh * N + n;
    float acc = 0.f;
    if (valid) {
        const uint4 a = o[row * TPR + part];
        const uint4 b = dout[row * TPR + part];
        const uint32_t av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float2 x = unpack2<BF16>(av[k]), y = unpack2<BF16>(bv[k]);
            acc = fmaf(x.x, y.x, acc);
            acc = fmaf(x.y, y.y, acc);
        }
        if (dqacc) {
            const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
            dqacc[(row * D + part * 8) / 4] = z;
            dqacc[(row * D + part * 8) / 4 + 1] = z;
        }
    }
#pragma unroll
    for (int off = TPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (bh < BH && part == 0) {
        float l2 = INFINITY;      // P = 2^(s - inf) = 0 for rows past N or with no visible key
        if (valid) {
            const float L = lse[row];
            if (L != -INFINITY) l2 = L * 1.4426950408889634f;
        }
        lse2[prow] = l2;
        dvec[prow] = valid ? acc : 0.f;
    }
}

// ---------------------------------------------------------------------------
// bwd_post: dQ = scale * dQacc in the 16-bit type
// ---------------------------------------------------------------------------
template <bool BF16>
__global__ void __launch_bounds__(256) bwd_post_kernel(const float4 *__restrict__ acc, uint4 *__restrict__ dq,
                                                       float scale, long long n8) {
    const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i >= n8) return;
    const float4 a = acc[2 * i], b = acc[2 * i + 1];
    dq[i] = make_uint4(pack2<BF16>(a.x * scale, a.y * scale), pack2<BF16>(a.z * scale, a.w * scale),
                       pack2<BF16>(b.x * scale, b.y * scale), pack2<BF16>(b.z * scale, b.w * scale));
}

// ---------------------------------------------------------------------------
// bwd_pre / bwd_post of packed variable-length batches: O, dO, dQ are packed
// [total_q][H][D], lse [H][total_q]; the statistics go to the padded
// [BH][Npad] layout of the key-block kernel (rows past a sequence's end:
// LSE * log2 e = +inf, D = 0, so that they add nothing), the accumulator is
// [H][total_q][D].
// ---------------------------------------------------------------------------
template <int D, bool BF16>
__global__ void __launch_bounds__(256)
    bwd_pre_varlen_kernel(const uint4 *__restrict__ o, const uint4 *__restrict__ dout, const float *__restrict__ lse,
                          float *__restrict__ lse2, float *__restrict__ dvec, float4 *__restrict__ dqacc,
                          const int *__restrict__ cu_q, int H, int total_q, int max_nq, int Npad, long long BH) {
    constexpr int TPR = D / 8;   // threads per row, 8 elements (16 bytes) each
    const long long tid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    const long long prow = tid / TPR;                 // padded row index bh * Npad + n
    const int part = static_cast<int>(tid % TPR);
    const long long bh = prow / Npad;
    const int n = static_cast<int>(prow % Npad);
    SeqSpan sq{0, 0};
    int h = 0;
    if (bh < BH) {
        const int b = static_cast<int>(bh / H);
        h = static_cast<int>(bh - static_cast<long long>(b) * H);
        sq = seq_span(cu_q, b, total_q, max_nq);
    }
    const bool valid = bh < BH && n < sq.len;
    const long long t = sq.start + n;                // packed row
    float acc = 0.f;
    if (valid) {
        const long long row = t * H + h;
        const uint4 a = o[row * TPR + part];
        const uint4 b = dout[row * TPR + part];
        const uint32_t av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float2 x = unpack2<BF16>(av[k]), y = unpack2<BF16>(bv[k]);
            acc = fmaf(x.x, y.x, acc);
            acc = fmaf(x.y, y.y, acc);
        }
        if (dqacc) {   // null: the deterministic backward keeps no accumulator
            const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
            const long long arow = static_cast<long long>(h) * total_q + t;
            dqacc[(arow * D + part * 8) / 4] = z;
            dqacc[(arow * D + part * 8) / 4 + 1] = z;
        }
    }
#pragma unroll
    for (int off = TPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (bh < BH && part == 0) {
        float l2 = INFINITY;      // P = 2^(s - inf) = 0 for rows past the sequence or with no visible key
        if (valid) {
            const float L = lse[static_cast<long long>(h) * total_q + t];
            if (L != -INFINITY) l2 = L * 1.4426950408889634f;
        }
        lse2[prow] = l2;
        dvec[prow] = valid ? acc : 0.f;
    }
}

// dq [total_q][H][D] = scale * dqacc [H][total_q][D], 8 elements per thread
template <int D, bool BF16>
__global__ void __launch_bounds__(256) bwd_post_varlen_kernel(const float4 *__restrict__ acc, uint4 *__restrict__ dq,
                                                              float scale, int H, int total_q) {
    constexpr int TPR = D / 8;
    const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;   // over [H][total_q][TPR]
    if (i >= static_cast<long long>(H) * total_q * TPR) return;
    const int part = static_cast<int>(i % TPR);
    const long long ht = i / TPR;
    const int h = static_cast<int>(ht / total_q);
    const long long t = ht - static_cast<long long>(h) * total_q;
    const float4 a = acc[2 * i], b = acc[2 * i + 1];
    dq[(t * H + h) * TPR + part] =
        make_uint4(pack2<BF16>(a.x * scale, a.y * scale), pack2<BF16>(a.z * scale, a.w * scale),
                   pack2<BF16>(b.x * scale, b.y * scale), pack2<BF16>(b.z * scale, b.w * scale));
}

// ---------------------------------------------------------------------------
// bwd_main
// ---------------------------------------------------------------------------
// GENERAL kernels handle Nq != Nk, windows and ALiBi through the visibility
// band; the others serve square problems (dense, causal, block-sparse) with
// the plain causal test, which keeps their inner loops as lean as possible.
template <int BM, bool GENERAL>
__device__ __forceinline__ bool qtile_kept(const BwdParams &p, int i, int j) {
    if (i >= p.nqt) return false;
    if constexpr (GENERAL) {
        const int q0 = i * BM, k0 = j * 128;
        const int q1 = min(q0 + BM - 1, p.Nq - 1), k1 = min(k0 + 127, p.Nk - 1);
        if (!band_any(q0, q1, k0, k1, p.off, p.wl, p.wr)) return false;
    } else {
        if ((p.mode & kCausal) && (i + 1) * BM <= j * 128) return false;   // every query precedes every key
    }
    if ((p.mode & kSparse) && p.mask[static_cast<size_t>((i * BM) / 128) * p.nkb + j] == 0) return false;
    return true;
}

// CTA blockIdx.x of a packed batch's backward grid, ordered sequence, key
// block, head (nkb: key blocks of the longest sequence): its (sequence, head)
// index b H + h and its key block.
__device__ __forceinline__ int packed_bh(int nkb, int H) {
    const unsigned per = static_cast<unsigned>(nkb) * static_cast<unsigned>(H);
    const unsigned b = blockIdx.x / per;
    return static_cast<int>(b * H + (blockIdx.x - b * per) % static_cast<unsigned>(H));
}
__device__ __forceinline__ int packed_j(int nkb, int H) {
    const unsigned per = static_cast<unsigned>(nkb) * static_cast<unsigned>(H);
    return static_cast<int>((blockIdx.x % per) / static_cast<unsigned>(H));
}

// Walks the query tiles that see key block j, in increasing order (warp-collective).
template <int BM, bool GENERAL>
struct QIter {
    int base = -32;
    uint32_t b = 0;
    __device__ __forceinline__ bool next(const BwdParams &p, int j, int &i) {
        while (b == 0u) {
            base += 32;
            if (base >= p.nqt) return false;
            b = __ballot_sync(0xffffffffu, qtile_kept<BM, GENERAL>(p, base + static_cast<int>(lane_id()), j));
        }
        const int k = __ffs(b) - 1;
        b &= b - 1;
        i = base + k;
        return true;
    }
};

// ---------------------------------------------------------------------------
// bwd_kernel (d = 64, 128): one CTA per 128-key block j, query tiles of 128.
//
// Every product is a full-rate tcgen05 shape (M = 128 or d, N = 128):
//   S^T  = K_j Q_i^T        SS    -> TMEM [0, 128)        (lane = key)
//   dP^T = V_j dO_i^T       SS    -> TMEM [128, 256)
//   dV  += P^T dO_i         TS    P^T (16-bit) written by the softmax-grad
//                                 warps over the S^T columns they have read
//   dK  += dS^T Q_i         SS    dS^T (16-bit) in shared memory
//   dQ_i^T = K_j^T dS^T     SS    -> TMEM [128, 256) once dP^T has been read
//                                 (lane = d; M = 64 at d = 64)
// dV, dK accumulate in TMEM [256, 256 + d) and [256 + d, 256 + 2 d).
//
// The softmax-grad work is split in two phases so that both overlap products:
//   A(i): P^T from S^T and LSE     (overlaps dK, dQ^T of the previous tile)
//   B(i): dS^T from dP^T, P and D  (overlaps dV(i) and S^T of the next tile)
// MMA issue order per tile i (i' = next kept tile):
//   [P(i) ready] dV(i), S^T(i') | [dS(i) ready] dK(i), dQ^T(i) |
//   [dQ^T(i) read out] dP^T(i')
// The tensor pipe completes in issue order, so S^T(i') may overwrite P^T(i)
// after dV(i), and dP^T(i') completing implies dK(i), dQ^T(i) have finished
// reading dS^T(i): one dS^T buffer suffices.
//
// Warp roles (512 threads, four warpgroups): warps 0-7 softmax-grad (warp w:
// TMEM lanes 32 (w % 4).., queries [64 (w / 4), +64)), then the dV / dK
// epilogue; warps 8-11 dQ drain (TMEM -> registers -> fp32 atomics into the
// accumulator); warp 12 TMA producer; warp 13 MMA issuer (owns TMEM); warps
// 14-15 idle.  The last warpgroup gives registers to the first three
// (setmaxnreg: 3 x 128 x 144 + 128 x 80 = 65536).
// ---------------------------------------------------------------------------
template <int D, int NS>
struct BwdCfg {
    static constexpr int BM = 128;                      // query rows per tile
    static constexpr int kKVTile = 128 * D * 2;         // K_j or V_j
    static constexpr int kChunk = 128 * 128;            // 64 columns of a 128-row tile (one swizzle atom wide)
    static constexpr int kQTile = BM * D * 2;           // Q_i or dO_i
    static constexpr int kKOff = 0;
    static constexpr int kVOff = kKOff + kKVTile;
    static constexpr int kQOff = kVOff + kKVTile;
    static constexpr int kdOOff = kQOff + NS * kQTile;
    static constexpr int kdSOff = kdOOff + NS * kQTile;   // dS^T: [2 query chunks][128 keys][64 queries]
    static constexpr int kStatBytes = BM * 4;
    static constexpr int kStatOff = kdSOff + 2 * kChunk;  // per stage: LSE log2 e [BM], D [BM]
    // d = 64: dQ of a query tile is staged as two halves [64 queries][64 d]
    // fp32 and added to the accumulator with bulk reductions (whole-line
    // requests; the per-lane reductions of an M = 64 product are 64 bytes)
    static constexpr int kDqHalf = 64 * D * 4;
    static constexpr int kDqStageOff = kStatOff + NS * 2 * kStatBytes;
    static constexpr int kDqStageBytes = D == 64 ? 2 * kDqHalf : 0;
    static constexpr int kBarOff = kDqStageOff + kDqStageBytes;
    static constexpr int kBarKV = 0;
    static constexpr int kBarQFull = 1;                   // Q_i and LSE_i landed
    static constexpr int kBarQEmpty = kBarQFull + NS;
    static constexpr int kBarOFull = kBarQEmpty + NS;     // dO_i and D_i landed
    static constexpr int kBarOEmpty = kBarOFull + NS;
    static constexpr int kBarSFull = kBarOEmpty + NS;     // S^T computed
    static constexpr int kBarDPFull = kBarSFull + 1;      // dP^T computed
    static constexpr int kBarPFull = kBarDPFull + 1;      // P^T in TMEM (256 arrivals)
    static constexpr int kBarDsFull = kBarPFull + 1;      // dS^T in smem, dP^T read (256 arrivals)
    static constexpr int kBarDqFull = kBarDsFull + 1;     // dQ^T computed
    static constexpr int kBarDqFree = kBarDqFull + 1;     // dQ^T read out (128 arrivals)
    static constexpr int kBarMmaDone = kBarDqFree + 1;
    static constexpr int kBarDqStageFree = kBarMmaDone + 1;   // d = 64: staging half free (issuing thread)
    static constexpr int kBarDqStaged = kBarDqStageFree + 1;  // d = 64: staging half written (128 arrivals)
    static constexpr int kNumBars = kBarDqStaged + 1;
    static constexpr int kMiscOff = kBarOff + kNumBars * 8;
    // No alignment slack: the kernel checks that dynamic shared memory starts
    // on a 1 KB boundary (the 128-byte swizzle atoms need it).
    static constexpr int kSmemBytes = kMiscOff + 16;
    static constexpr int kThreads = 512;
    static constexpr int kRegsWork = 144;               // warpgroups 0-2 after setmaxnreg
    static constexpr int kRegsCtl = 80;                  // warpgroup 3
    static_assert(3 * 128 * kRegsWork + 128 * kRegsCtl <= 65536, "register split");
    static constexpr int kWarpTma = 12;
    static constexpr int kWarpMma = 13;
    static constexpr int kColS = 0;
    static constexpr int kColDP = 128;
    static constexpr int kColDV = 256;
    static constexpr int kColDK = 256 + D;
    // dQ^T: its own columns at d = 64 (free there), so dP^T of the next tile
    // need not wait for the drain; at d = 128 it reuses the dP^T columns
    static constexpr int kColDQ = D == 64 ? 384 : kColDP;
    static_assert(D == 64 || D == 128, "head dim");
    static_assert(kSmemBytes <= 227 * 1024, "shared memory");
};

constexpr int kErrSmemAlign = 5;   // matches FA_ERR_CUDA

template <int D, int NS, bool BF16, bool GENERAL, bool VARLEN = false>
__global__ void __launch_bounds__(512, 1)
    bwd_kernel(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
               const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmdo,
               const __grid_constant__ CUtensorMap tmdk, const __grid_constant__ CUtensorMap tmdv,
               const BwdParams p) {
    using C = BwdCfg<D, NS>;
    constexpr int BM = C::BM;
    static_assert(GENERAL || !VARLEN, "packed batches use the general band");
    // one-dimensional grid, (batch, head) minor: causal runs the heaviest key
    // blocks (j = 0) of every (b, h) first (longest work first).  Packed
    // batches: sequence major, then key blocks, heads minor, so that the
    // running CTAs reduce into the dQ rows of one or two sequences, which stay
    // in L2 (in the (b, h)-minor order every sequence's rows are live at once)
    const int bh = VARLEN ? packed_bh(p.nkb, p.H) : static_cast<int>(blockIdx.x % static_cast<unsigned>(p.nbh));
    const int j = VARLEN ? packed_j(p.nkb, p.H) : static_cast<int>(blockIdx.x / static_cast<unsigned>(p.nbh));
    // packed variable-length batches: the grid is sized by the longest
    // sequence; a CTA past its own sequence's keys leaves before any setup.
    // lp is p with this sequence's lengths; TMA rows are offset by qrow0 /
    // krow0 in plane (the head)
    BwdParams lp;
    int qrow0 = 0, krow0 = 0, plane = bh;
    if constexpr (VARLEN) {
        const int b = bh / p.H;
        plane = bh - b * p.H;
        const SeqSpan sq = seq_span(p.cu_q, b, p.total_q, p.Nq);
        const SeqSpan sk = seq_span(p.cu_k, b, p.total_k, p.Nk);
        if (j * 128 >= sk.len) return;
        lp = p;
        lp.Nq = sq.len;
        lp.Nk = sk.len;
        lp.nqt = (sq.len + BM - 1) / BM;
        lp.nkb = (sk.len + 127) / 128;
        lp.off = sk.len - sq.len;
        qrow0 = sq.start;
        krow0 = sk.start;
    }
    const BwdParams &ip = pick<VARLEN>(lp, p);
    // accumulator row of this (b, h)'s query row q
    auto dq_row = [&](int q) -> size_t {
        if constexpr (VARLEN) return static_cast<size_t>(plane) * p.total_q + qrow0 + q;
        else return static_cast<size_t>(bh) * p.Nq + q;
    };
    extern __shared__ __align__(1024) uint8_t smem_buf[];
    if (smem_u32(smem_buf) & 1023u) {
        if (threadIdx.x == 0) atomicCAS(&g_dev_status, 0, kErrSmemAlign);
        return;
    }
    uint8_t *smem = smem_buf;
    const uint32_t sbase = smem_u32(smem);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    auto bar = [&](int i) -> uint32_t { return sbase + C::kBarOff + 8u * i; };
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + C::kMiscOff);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::kMiscOff + 4);

    if (threadIdx.x == 0) {
        mbar_init(bar(C::kBarKV), 1);
        for (int s = 0; s < NS; ++s) {
            mbar_init(bar(C::kBarQFull + s), 1);
            mbar_init(bar(C::kBarQEmpty + s), 1);
            mbar_init(bar(C::kBarOFull + s), 1);
            mbar_init(bar(C::kBarOEmpty + s), 1);   // dP^T(i) and dV(i) have read dO_i
        }
        mbar_init(bar(C::kBarSFull), 1);
        mbar_init(bar(C::kBarDPFull), 1);
        mbar_init(bar(C::kBarPFull), 256);
        mbar_init(bar(C::kBarDsFull), 256);
        mbar_init(bar(C::kBarDqFull), 1);
        mbar_init(bar(C::kBarDqFree), 128);
        mbar_init(bar(C::kBarMmaDone), 1);
        mbar_init(bar(C::kBarDqStageFree), 1);
        mbar_init(bar(C::kBarDqStaged), 128);
        *abort_flag = 0;
        mbar_fence_init();
    }
    if (warp == C::kWarpMma) {
        tmem_alloc(smem_u32(tmem_holder), 512);
        tmem_relinquish();
    }
    if (warp == C::kWarpTma && lane == 0) {
        tma_prefetch_desc(&tmk);
        tma_prefetch_desc(&tmv);
        tma_prefetch_desc(&tmq);
        tma_prefetch_desc(&tmdo);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    int cnt = 0;        // query tiles processed by this warp's role
    bool ok = true;

    if (warp >= 12) {
        setmaxnreg_dec<C::kRegsCtl>();
        if (warp == C::kWarpTma) {
            // ------------------------------------------------------------ producer
            if (lane == 0) {
                mbar_arrive_expect_tx(bar(C::kBarKV), 2 * C::kKVTile);
                for (int c = 0; c < D / 64; ++c) {
                    tma_load_3d(sbase + C::kKOff + c * C::kChunk, &tmk, bar(C::kBarKV), c * 64, krow0 + j * 128,
                                plane);
                    tma_load_3d(sbase + C::kVOff + c * C::kChunk, &tmv, bar(C::kBarKV), c * 64, krow0 + j * 128,
                                plane);
                }
            }
            __syncwarp();
            QIter<BM, GENERAL> it;
            int i;
            while (it.next(ip, j, i)) {
                const int s = cnt % NS;
                // Q_i with the padded LSE_i, dO_i with D_i (TMA tiles and bulk
                // copies of the statistics prepared by bwd_pre), each pair on
                // its own transaction barrier
                const size_t srow = static_cast<size_t>(bh) * p.Npad + static_cast<size_t>(i) * BM;
                const uint32_t st = sbase + C::kStatOff + s * 2 * C::kStatBytes;
                ok = wait_bar(bar(C::kBarQEmpty + s), ((cnt / NS) & 1) ^ 1u, abort_flag);
                if (!ok) break;
                if (lane == 0) {
                    const uint32_t qb = bar(C::kBarQFull + s);
                    mbar_arrive_expect_tx(qb, C::kQTile + C::kStatBytes);
                    for (int c = 0; c < D / 64; ++c)
                        tma_load_3d(sbase + C::kQOff + s * C::kQTile + c * C::kChunk, &tmq, qb, c * 64,
                                    qrow0 + i * BM, plane);
                    bulk_load(st, p.lse2 + srow, C::kStatBytes, qb);
                }
                __syncwarp();
                ok = wait_bar(bar(C::kBarOEmpty + s), ((cnt / NS) & 1) ^ 1u, abort_flag);
                if (!ok) break;
                if (lane == 0) {
                    const uint32_t ob = bar(C::kBarOFull + s);
                    mbar_arrive_expect_tx(ob, C::kQTile + C::kStatBytes);
                    for (int c = 0; c < D / 64; ++c)
                        tma_load_3d(sbase + C::kdOOff + s * C::kQTile + c * C::kChunk, &tmdo, ob, c * 64,
                                    qrow0 + i * BM, plane);
                    bulk_load(st + C::kStatBytes, p.dvec + srow, C::kStatBytes, ob);
                }
                __syncwarp();
                ++cnt;
            }
            drain_bar(bar(C::kBarKV), 0);
            for (int x = (cnt > NS ? cnt - NS : 0); x < cnt; ++x) {
                drain_bar(bar(C::kBarQFull + x % NS), (x / NS) & 1);
                drain_bar(bar(C::kBarOFull + x % NS), (x / NS) & 1);
            }
        } else if (warp == C::kWarpMma) {
            // ------------------------------------------------------------ MMA issuer
            const uint32_t leader = elect_one();   // the lane that issues tcgen05 ops
            constexpr uint32_t kIdS = instr_desc_f16(128, BM, BF16, false, false);   // S^T, dP^T
            constexpr uint32_t kIdKV = instr_desc_f16(128, D, BF16, false, true);    // dV, dK
            constexpr uint32_t kIdQ = instr_desc_f16(D, BM, BF16, true, true);       // dQ^T
            // descriptors built once; each instruction only offsets the start address
            const SmemDesc dK_k = make_desc(sbase + C::kKOff, 16, 1024);
            const SmemDesc dV_k = make_desc(sbase + C::kVOff, 16, 1024);
            const SmemDesc dQ_k = make_desc(sbase + C::kQOff, 16, 1024);
            const SmemDesc ddO_k = make_desc(sbase + C::kdOOff, 16, 1024);
            const SmemDesc dQ_mn = make_desc(sbase + C::kQOff, C::kChunk, 1024);
            const SmemDesc ddO_mn = make_desc(sbase + C::kdOOff, C::kChunk, 1024);
            const SmemDesc ddS_k = make_desc(sbase + C::kdSOff, 16, 1024);
            const SmemDesc ddS_mn = make_desc(sbase + C::kdSOff, C::kChunk, 1024);
            const SmemDesc dK_mn = make_desc(sbase + C::kKOff, C::kChunk, 1024);
            auto issue_s = [&](int s) {          // S^T = K_j Q_i^T
#pragma unroll
                for (int k = 0; k < D / 16; ++k) {
                    const uint32_t o = (k >> 2) * C::kChunk + (k & 3) * 32;
                    mma_ss(tmem + C::kColS, dK_k.at(o), dQ_k.at(s * C::kQTile + o), kIdS, k > 0 ? 1u : 0u, leader);
                }
            };
            auto issue_dp = [&](int s) {         // dP^T = V_j dO_i^T
#pragma unroll
                for (int k = 0; k < D / 16; ++k) {
                    const uint32_t o = (k >> 2) * C::kChunk + (k & 3) * 32;
                    mma_ss(tmem + C::kColDP, dV_k.at(o), ddO_k.at(s * C::kQTile + o), kIdS, k > 0 ? 1u : 0u, leader);
                }
            };
            auto issue_dv = [&](int s, bool acc) {   // dV += P^T dO_i; P^T of queries 16k.. at column 8k + 32 (k / 4)
#pragma unroll
                for (int k = 0; k < BM / 16; ++k)
                    mma_ts(tmem + C::kColDV, tmem + C::kColS + 8 * k + 32 * (k >> 2), ddO_mn.at(s * C::kQTile + k * 2048),
                           kIdKV, (acc || k > 0) ? 1u : 0u, leader);
            };
            const bool with_dq = p.dqacc != nullptr;   // else the deterministic dQ pass computes dQ
            auto issue_dk_dq = [&](int s, bool acc) {
#pragma unroll
                for (int k = 0; k < BM / 16; ++k)    // dK += dS^T Q_i
                    mma_ss(tmem + C::kColDK, ddS_k.at((k >> 2) * C::kChunk + (k & 3) * 32),
                           dQ_mn.at(s * C::kQTile + k * 2048), kIdKV, (acc || k > 0) ? 1u : 0u, leader);
                if (with_dq) {
#pragma unroll
                    for (int k = 0; k < 8; ++k)      // dQ^T (D x BM) = K_j^T dS^T, over the 128 keys
                        mma_ss(tmem + C::kColDQ, dK_mn.at(k * 2048), ddS_mn.at(k * 2048), kIdQ, k > 0 ? 1u : 0u,
                               leader);
                }
            };

            QIter<BM, GENERAL> it;
            int i, in;
            bool have = it.next(ip, j, i);
            if (have) {
                ok = wait_bar(bar(C::kBarKV), 0, abort_flag) && wait_bar(bar(C::kBarQFull), 0, abort_flag);
                if (ok) {
                    tc_fence_after();
                    issue_s(0);
                    mma_commit(bar(C::kBarSFull), leader);
                    __syncwarp();
                    ok = wait_bar(bar(C::kBarOFull), 0, abort_flag);
                }
                if (ok) {
                    tc_fence_after();
                    issue_dp(0);
                    mma_commit(bar(C::kBarDPFull), leader);
                    __syncwarp();
                }
            }
            while (ok && have) {
                const int s = cnt % NS;
                const int sn = (cnt + 1) % NS;
                const uint32_t ph = cnt & 1;
                const bool have_n = it.next(ip, j, in);
                ok = wait_bar(bar(C::kBarPFull), ph, abort_flag);
                if (!ok) break;
                tc_fence_after();
                issue_dv(s, cnt > 0);
                mma_commit(bar(C::kBarOEmpty + s), leader);   // dP^T(i), dV(i): the readers of dO_i
                __syncwarp();
                if (have_n) {
                    ok = wait_bar(bar(C::kBarQFull + sn), ((cnt + 1) / NS) & 1, abort_flag);
                    if (!ok) break;
                    tc_fence_after();
                    {
                        issue_s(sn);
                        mma_commit(bar(C::kBarSFull), leader);
                    }
                    __syncwarp();
                }
                ok = wait_bar(bar(C::kBarDsFull), ph, abort_flag);
                if (!ok) break;
                if (D == 64 && with_dq && cnt > 0) {
                    // dQ^T has its own columns: the drain must have read out the previous tile's
                    ok = wait_bar(bar(C::kBarDqFree), (cnt - 1) & 1, abort_flag);
                    if (!ok) break;
                }
                tc_fence_after();
                {
                    issue_dk_dq(s, cnt > 0);
                    if (with_dq) mma_commit(bar(C::kBarDqFull), leader);
                    mma_commit(bar(C::kBarQEmpty + s), leader);
                }
                __syncwarp();
                if (have_n) {
                    // the dP^T columns are free once dS(i) is in place, unless
                    // dQ^T(i) was written over them (d = 128): then once the
                    // drain has read it out
                    ok = !with_dq || D == 64 || wait_bar(bar(C::kBarDqFree), ph, abort_flag);
                    if (!ok) break;
                    ok = wait_bar(bar(C::kBarOFull + sn), ((cnt + 1) / NS) & 1, abort_flag);
                    if (!ok) break;
                    tc_fence_after();
                    {
                        issue_dp(sn);
                        mma_commit(bar(C::kBarDPFull), leader);
                    }
                    __syncwarp();
                }
                ++cnt;
                have = have_n;
                i = in;
            }
            mma_commit(bar(C::kBarMmaDone), leader);
            __syncwarp();
            drain_bar(bar(C::kBarMmaDone), 0);
        }
    } else {
        setmaxnreg_inc<C::kRegsWork>();
        if (warp < 8) {
            // ------------------------------------------------------------ softmax-grad
            const int qd = warp & 3;            // TMEM lane quadrant
            const int qh = warp >> 2;           // query half
            const uint32_t lane_off = static_cast<uint32_t>(qd * 32) << 16;
            const int r = qd * 32 + lane;       // key row within the block
            const int key = j * 128 + r;
            const float c = p.scale_log2;
            QIter<BM, GENERAL> it;
            int i;
            while (it.next(ip, j, i)) {
                const int s = cnt % NS;
                const uint32_t ph = cnt & 1;
                ok = wait_bar(bar(C::kBarSFull), ph, abort_flag) &&
                     wait_bar(bar(C::kBarQFull + s), (cnt / NS) & 1, abort_flag);
                if (!ok) break;
                tc_fence_after();
                const float4 *lse4 = reinterpret_cast<const float4 *>(smem + C::kStatOff + s * 2 * C::kStatBytes);
                const float4 *dd4 = lse4 + BM / 4;
                // phase A: P^T = 2^(S^T * scale * log2 e - LSE * log2 e), masked,
                // rounded to 16 bits (kept packed in registers for phase B) and
                // written over the S^T columns already read
                const int q0 = 64 * qh;
                // queries q0 + kk of this thread's half that see key `key`: lo <= kk <= hi
                // (key q + off - wl .. q + off + wr); keys past Nk see none
                int qk, lo, hi;
                bool masked;
                if constexpr (GENERAL) {
                    qk = key - ip.off - (i * BM + q0);     // |values| < 2^30 (Nq, Nk <= 2^28)
                    lo = max(qk - p.wr, -1);
                    hi = min(qk + p.wl, 64);
                    if (key >= ip.Nk) lo = 64;
                    masked = __any_sync(0xffffffffu, lo > 0 || hi < 63);
                } else {
                    // square: the diagonal tile hides queries before the key
                    qk = 0;
                    hi = 64;
                    lo = r - q0;
                    masked = (p.mode & kCausal) && i == j;
                }
                uint32_t pk[32];
                {
                    uint32_t sr[64];
                    tmem_ld32(tmem + lane_off + C::kColS + q0, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
                    tmem_ld32(tmem + lane_off + C::kColS + q0 + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
                    tmem_wait_ld(sr);
                    if (GENERAL && p.alibi) {
                        // score + bias / scale, bias = -slope |q + off - key|
                        const float sl = -p.alibi[bh % p.H] / p.scale;
                        const float base = static_cast<float>(-qk);
#pragma unroll
                        for (int kk = 0; kk < 64; ++kk)
                            sr[kk] = __float_as_uint(fmaf(sl, fabsf(base + static_cast<float>(kk)), __uint_as_float(sr[kk])));
                    }
#pragma unroll
                    for (int k4 = 0; k4 < 16; ++k4) {
                        const float4 l4 = lse4[q0 / 4 + k4];
                        float x0 = ex2(fmaf(__uint_as_float(sr[4 * k4]), c, -l4.x));
                        float x1 = ex2(fmaf(__uint_as_float(sr[4 * k4 + 1]), c, -l4.y));
                        float x2 = ex2(fmaf(__uint_as_float(sr[4 * k4 + 2]), c, -l4.z));
                        float x3 = ex2(fmaf(__uint_as_float(sr[4 * k4 + 3]), c, -l4.w));
                        pk[2 * k4] = pack2<BF16>(x0, x1);
                        pk[2 * k4 + 1] = pack2<BF16>(x2, x3);
                    }
                }
                if (masked) {
                    // zero the 16-bit P of queries outside [lo, hi] (element 2k in the low half)
#pragma unroll
                    for (int k = 0; k < 32; ++k) {
                        uint32_t keep = 0xffffffffu;
                        if (2 * k < lo || 2 * k > hi) keep &= 0xffff0000u;
                        if (2 * k + 1 < lo || 2 * k + 1 > hi) keep &= 0x0000ffffu;
                        pk[k] &= keep;
                    }
                }
                tmem_st32(tmem + lane_off + C::kColS + q0, pk);
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(bar(C::kBarPFull));
                // phase B: dS^T = P^T o (dP^T - D), with the 16-bit P^T
                ok = wait_bar(bar(C::kBarDPFull), ph, abort_flag) &&
                     wait_bar(bar(C::kBarOFull + s), (cnt / NS) & 1, abort_flag);   // D_i
                if (!ok) break;
                tc_fence_after();
                {
                    uint32_t pr[64];
                    tmem_ld32(tmem + lane_off + C::kColDP + q0, *reinterpret_cast<uint32_t(*)[32]>(&pr[0]));
                    tmem_ld32(tmem + lane_off + C::kColDP + q0 + 32, *reinterpret_cast<uint32_t(*)[32]>(&pr[32]));
                    tmem_wait_ld(pr);
                    // row r of a K-major [128 keys][64 queries] 128B-swizzled tile
                    uint8_t *sdS = smem + C::kdSOff + qh * C::kChunk + r * 128;
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        uint32_t dk[4];
#pragma unroll
                        for (int h2 = 0; h2 < 2; ++h2) {
                            const int k4 = 2 * u + h2;
                            const float4 d4 = dd4[q0 / 4 + k4];
                            const float2 p01 = unpack2<BF16>(pk[2 * k4]), p23 = unpack2<BF16>(pk[2 * k4 + 1]);
                            dk[2 * h2] = pack2<BF16>(p01.x * (__uint_as_float(pr[4 * k4]) - d4.x),
                                                     p01.y * (__uint_as_float(pr[4 * k4 + 1]) - d4.y));
                            dk[2 * h2 + 1] = pack2<BF16>(p23.x * (__uint_as_float(pr[4 * k4 + 2]) - d4.z),
                                                         p23.y * (__uint_as_float(pr[4 * k4 + 3]) - d4.w));
                        }
                        *reinterpret_cast<uint4 *>(sdS + ((u ^ (r & 7)) << 4)) = make_uint4(dk[0], dk[1], dk[2], dk[3]);
                    }
                }
                tc_fence_before();
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                mbar_arrive(bar(C::kBarDsFull));
                ++cnt;
            }
            // ------------------------------------------------------------ dV / dK epilogue
            {
                // dV (warps 0-3) and dK (warps 4-7) are staged as 128-byte-swizzled
                // 64-column chunks in the V_j / K_j buffers (free once every
                // product has completed) and written by TMA stores
                bool done = ok;
                if (done && cnt > 0) done = wait_bar(bar(C::kBarMmaDone), 0, abort_flag);
                tc_fence_after();
                const bool is_dv = warp < 4;
                const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
                const int r = (warp & 3) * 32 + lane;
                const float mul = is_dv ? 1.0f : p.scale;
                uint8_t *stage = smem + (is_dv ? C::kVOff : C::kKOff);
                const uint32_t col0 = is_dv ? C::kColDV : C::kColDK;
                // a key block that no query tile sees never waited for its K/V
                // loads: they must land before the staging areas are written
                if (done && cnt == 0) drain_bar(bar(C::kBarKV), 0);
                // packed batches: a key block that ends inside the next
                // sequence's rows is written row by row with plain stores (a
                // TMA store clips only at the end of the tensor)
                const int krows = VARLEN ? ip.Nk - j * 128 : 128;
                if (done) {
        #pragma unroll 1
                    for (int ch = 0; ch < D / 32; ++ch) {
                        uint32_t v[32];
                        if (cnt > 0) {
                            tmem_ld32_wait(tmem + lane_off + col0 + 32 * ch, v);
                        } else {
    #pragma unroll
                            for (int k = 0; k < 32; ++k) v[k] = 0u;   // no query sees this key block
                        }
                        uint32_t pk[16];
    #pragma unroll
                        for (int k = 0; k < 16; ++k)
                            pk[k] = pack2<BF16>(__uint_as_float(v[2 * k]) * mul, __uint_as_float(v[2 * k + 1]) * mul);
                        if (VARLEN && krows < 128) {
                            if (r < krows) {
                                uint4 *g = reinterpret_cast<uint4 *>(
                                    static_cast<uint8_t *>(is_dv ? p.dv : p.dk) +
                                    (static_cast<size_t>(krow0 + j * 128 + r) * p.H + plane) * (D * 2) + ch * 64);
    #pragma unroll
                                for (int k = 0; k < 4; ++k)
                                    g[k] = make_uint4(pk[4 * k], pk[4 * k + 1], pk[4 * k + 2], pk[4 * k + 3]);
                            }
                            continue;
                        }
                        uint8_t *srow = stage + (ch >> 1) * C::kChunk + r * 128;
    #pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const int u = (ch & 1) * 4 + k;
                            *reinterpret_cast<uint4 *>(srow + ((u ^ (r & 7)) << 4)) =
                                make_uint4(pk[4 * k], pk[4 * k + 1], pk[4 * k + 2], pk[4 * k + 3]);
                        }
                    }
                }
                fence_async_smem();
                named_sync(is_dv ? 1 : 2, 128);   // the four warps of this output (every one gets here)
                if (done && krows >= 128 && (warp & 3) == 0 && lane == 0) {
                    for (int c = 0; c < D / 64; ++c)   // keys >= Nk are clipped
                        tma_store_3d(is_dv ? &tmdv : &tmdk, smem_u32(stage + c * C::kChunk), c * 64,
                                     krow0 + j * 128, plane);
                    bulk_commit();
                    bulk_wait_read();
                }
            }
        } else {
            // ------------------------------------------------------------ dQ drain
            // dQ^T rows are d indices.  At d = 128 every TMEM lane is a row; at
            // d = 64 (an M = 64 product) row m sits in lane 32 (m / 16) + m % 16.
            const int wq = warp & 3;
            const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
            const bool row_lane = (D == 128) || (lane < 16);
            const int dcol = (D == 128) ? wq * 32 + lane : wq * 16 + (lane & 15);
            const bool issuer = wq == 0 && lane == 0;   // d = 64: issues the bulk reductions
            int nh = 0;                                  // d = 64: staged halves
            QIter<BM, GENERAL> it;
            int i;
            while (p.dqacc != nullptr && it.next(ip, j, i)) {
                ok = wait_bar(bar(C::kBarDqFull), cnt & 1, abort_flag);
                if (!ok) break;
                tc_fence_after();
                uint32_t v[BM];
                // 128 registers: four loads and one wait (a single load-and-wait
                // statement does not fit this kernel's register budget); the
                // wait names every loaded register
#pragma unroll
                for (int ch = 0; ch < BM / 32; ++ch)
                    tmem_ld32(tmem + lane_off + C::kColDQ + 32 * ch, *reinterpret_cast<uint32_t(*)[32]>(&v[32 * ch]));
                tmem_wait_ld(v);
                tc_fence_before();
                mbar_arrive(bar(C::kBarDqFree));
                if constexpr (D == 64) {
                    // two halves of 64 queries: [64 queries][64 d] fp32 in the
                    // staging half h, then one bulk reduction of the contiguous
                    // rows into the accumulator (unrolled: v is indexed by h).
                    // The four drain warps hand over through mbarriers with
                    // bounded waits, so that none can be left waiting.
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int q0 = i * BM + 64 * h;
                        const int rows = min(64, ip.Nq - q0);
                        if (rows <= 0) break;
                        // staging half h was last read by the reduction two before
                        if (issuer) {
                            bulk_wait_read_1();
                            mbar_arrive(bar(C::kBarDqStageFree));
                        }
                        ok = wait_bar(bar(C::kBarDqStageFree), nh & 1, abort_flag);
                        if (!ok) break;
                        if (row_lane) {
                            float *st = reinterpret_cast<float *>(smem + C::kDqStageOff + h * C::kDqHalf) + dcol;
#pragma unroll
                            for (int k = 0; k < 64; ++k) st[k * D] = __uint_as_float(v[64 * h + k]);
                        }
                        fence_async_smem();
                        mbar_arrive(bar(C::kBarDqStaged));
                        if (wq == 0) {
                            ok = wait_bar(bar(C::kBarDqStaged), nh & 1, abort_flag);
                            if (!ok) break;
                            if (issuer) {
                                bulk_reduce_add_f32(p.dqacc + dq_row(q0) * D,
                                                    sbase + C::kDqStageOff + h * C::kDqHalf,
                                                    static_cast<uint32_t>(rows) * D * 4);
                                bulk_commit();
                            }
                        }
                        ++nh;
                    }
                    if (!ok) break;
                } else if (row_lane) {
                    float *acc = p.dqacc + dq_row(i * BM) * D + dcol;
                    const int lim = ip.Nq - i * BM;
#pragma unroll
                    for (int k = 0; k < BM; ++k)
                        if (k < lim) atomicAdd(acc + k * D, __uint_as_float(v[k]));
                }
                ++cnt;
            }
            // the staged dQ must be read, and added, before the CTA exits
            if (D == 64 && issuer) bulk_wait_all();
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == C::kWarpMma) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// Workspace: lse2 [BH][Npad] and D [BH][Npad] fp32 (Npad = N rounded up to
// 128), then the fp32 dQ accumulator [BH][N][d].
inline int bwd_npad(int N) { return (N + 127) / 128 * 128; }
inline size_t bwd_workspace_bytes(long long BH, int N, int d) {
    return 2 * static_cast<size_t>(BH) * bwd_npad(N) * 4 + static_cast<size_t>(BH) * N * d * 4;
}

}  // namespace fa
