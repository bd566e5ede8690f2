// fa_bwd_dq.cuh -- the dQ pass of the deterministic backward, sm_100a.
//
// The default backward adds the dQ contribution of every key block into an
// fp32 accumulator with atomics, so the low bits of dQ depend on the order in
// which CTAs finish.  A fully deterministic backward is slower
// ("FlashAttention 深度解析" section 五 lists it among the engineering limits);
// here it is built as two sweeps:
//   * the key-block kernel (bwd_kernel / bwd_split_kernel) with its dQ
//     product and atomic drain switched off: dK and dV only;
//   * this kernel: one CTA per 128-row query tile i sweeps the key blocks j
//     the tile sees, in increasing order, and sums
//         dQ_i = scale * sum_j dS_ij K_j,   dS_ij = P_ij o (dP_ij - D_i),
//         P_ij = exp(scale Q_i K_j^T - LSE_i),   dP_ij = dO_i V_j^T
//     in tensor memory, always in the same order, then rounds it once.
// No atomics and no fp32 accumulator: dQ is bitwise reproducible.  S and dP
// are recomputed (the key-block kernel computes them as well), so the pass
// costs three of the five backward products again.
//
// Products (M = 128 query rows, lane = query row):
//   S  = Q_i K_j^T      SS  -> an S buffer in TMEM
//   dP = dO_i V_j^T     SS  -> TMEM [256, 384)
//   dQ += dS K_j        TS  dS (16-bit), written by the softmax-grad warps over
//                           the S columns they have read; dQ accumulates in TMEM
// d = 64, 128: two S buffers [0, 128), [128, 256), dQ at [384, 384 + d), K_j
//   and V_j in rings of whole tiles.  Issue order per key block c:
//     [dP(c) read] dP(c + 1) | [dS(c) ready] dQ(c), S(c + 2)
//   so the tensor pipe computes dP(c + 1), dQ(c) and S(c + 2) while the
//   softmax-grad warps work on block c + 1.
// d = 256: dQ needs 256 columns, so one S buffer at [0, 128); K_j is held as
//   two halves (d columns [0, 128) and [128, 256)), V_j streams in 64-column
//   chunks.  Issue order: [dS(c) ready] dQ(c) half 0, half 1, S(c + 1),
//   dP(c + 1); K_{c+1} half 0 lands while dQ(c) half 1 runs.
// The tensor pipe completes in issue order, so an S product may overwrite the
// dS that the dQ product issued before it reads.
//
// Warp roles (352 threads): warps 0-7 softmax-grad (warp w: TMEM lanes
// 32 (w % 4).. = query rows, keys [64 (w / 4), +64) of each block), then the
// dQ epilogue; warp 8 TMA for Q_i, dO_i and K; warp 9 MMA issuer (owns TMEM);
// warp 10 TMA for V.
#pragma once

#include "fa_bwd.cuh"

namespace fa {

template <int D>
struct DqCfg {
    static constexpr bool kWide = D == 256;
    static constexpr int NSK = D == 64 ? 4 : (D == 128 ? 3 : 1);   // K stages (whole tiles)
    static constexpr int NSV = D == 64 ? 3 : 2;                      // V stages (tiles; 64-column chunks at d = 256)
    static constexpr int kChunk = 128 * 128;                         // 64 columns of a 128-row tile
    static constexpr int kTile = 128 * D * 2;                        // a 128-row tile of Q, dO, K or V
    static constexpr int kVSlot = kWide ? kChunk : kTile;
    static constexpr int kQOff = 0;
    static constexpr int kdOOff = kTile;
    static constexpr int kKOff = 2 * kTile;
    static constexpr int kVOff = kKOff + NSK * kTile;
    static constexpr int kBarOff = kVOff + NSV * kVSlot;
    static constexpr int kKBars = kWide ? 2 : NSK;                   // d = 256: one barrier pair per K half
    static constexpr int kSBufs = kWide ? 1 : 2;
    static constexpr int kBarQ = 0;
    static constexpr int kBarKFull = 1;
    static constexpr int kBarKEmpty = kBarKFull + kKBars;
    static constexpr int kBarVFull = kBarKEmpty + kKBars;
    static constexpr int kBarVEmpty = kBarVFull + NSV;
    static constexpr int kBarSFull = kBarVEmpty + NSV;               // per S buffer: S computed
    static constexpr int kBarDsFull = kBarSFull + kSBufs;            // per S buffer: dS written (256 arrivals)
    static constexpr int kBarDPFull = kBarDsFull + kSBufs;
    static constexpr int kBarDPFree = kBarDPFull + 1;                // dP read out (256 arrivals)
    static constexpr int kBarMmaDone = kBarDPFree + 1;
    static constexpr int kNumBars = kBarMmaDone + 1;
    static constexpr int kMiscOff = kBarOff + kNumBars * 8;
    static constexpr int kSmemBytes = kMiscOff + 16 + 1024;          // + slack for 1 KB alignment
    static constexpr int kThreads = 352;
    static constexpr int kWarpTmaK = 8;
    static constexpr int kWarpMma = 9;
    static constexpr int kWarpTmaV = 10;
    static constexpr int kColS = 0;                                  // S buffer b at 128 b
    static constexpr int kColDP = kWide ? 128 : 256;
    static constexpr int kColDQ = kWide ? 256 : 384;
    static_assert(D == 64 || D == 128 || D == 256, "head dim");
    static_assert(kColDQ + D <= 512, "TMEM columns");
    static_assert(kSmemBytes <= 227 * 1024, "shared memory");
};

// Key block j holds a key that some query of the 128-row tile i sees.
template <bool GENERAL>
__device__ __forceinline__ bool kblock_kept(const BwdParams &p, int i, int j) {
    if (j >= p.nkb) return false;
    if constexpr (GENERAL) {
        const int q0 = i * 128, k0 = j * 128;
        const int q1 = min(q0 + 127, p.Nq - 1), k1 = min(k0 + 127, p.Nk - 1);
        if (!band_any(q0, q1, k0, k1, p.off, p.wl, p.wr)) return false;
    } else {
        if ((p.mode & kCausal) && j > i) return false;   // every key follows every query
    }
    if ((p.mode & kSparse) && p.mask[static_cast<size_t>(i) * p.nkb + j] == 0) return false;
    return true;
}

// Walks the key blocks that query tile i sees, in increasing order (warp-collective).
template <bool GENERAL>
struct KIter {
    int base = -32;
    uint32_t b = 0;
    __device__ __forceinline__ bool next(const BwdParams &p, int i, int &j) {
        while (b == 0u) {
            base += 32;
            if (base >= p.nkb) return false;
            b = __ballot_sync(0xffffffffu, kblock_kept<GENERAL>(p, i, base + static_cast<int>(lane_id())));
        }
        const int k = __ffs(b) - 1;
        b &= b - 1;
        j = base + k;
        return true;
    }
};

// p.nqt counts 128-row query tiles here; p.dq receives dQ (16-bit, [BH][Nq][D]).
template <int D, bool BF16, bool GENERAL, bool VARLEN = false>
__global__ void __launch_bounds__(352, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                  const __grid_constant__ CUtensorMap tmv, const __grid_constant__ CUtensorMap tmdo,
                  const __grid_constant__ CUtensorMap tmdq, const BwdParams p) {
    using C = DqCfg<D>;
    constexpr int NSK = C::NSK;
    constexpr int NSV = C::NSV;
    constexpr int NSB = C::kSBufs;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = smem_u32(smem);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    static_assert(GENERAL || !VARLEN, "packed batches use the general band");
    // one-dimensional grid, (batch, head) minor; the last query tiles see the
    // most keys (causal, bottom-right bands), so they start first.  Packed
    // batches: sequence major, then query tiles from the last, heads minor;
    // a CTA past its own sequence's query tiles leaves before any setup.
    // lp is p with the sequence's lengths; TMA rows are offset by qrow0 /
    // krow0 in plane (the head)
    int bh, i;
    BwdParams lp;
    int qrow0 = 0, krow0 = 0, plane = 0;
    if constexpr (VARLEN) {
        const unsigned per = static_cast<unsigned>(p.nqt) * static_cast<unsigned>(p.H);
        const int b = static_cast<int>(blockIdx.x / per);
        const int r = static_cast<int>(blockIdx.x - b * per);
        const int ii = r / p.H;
        plane = r - ii * p.H;
        bh = b * p.H + plane;
        const SeqSpan sq = seq_span(p.cu_q, b, p.total_q, p.Nq);
        const SeqSpan sk = seq_span(p.cu_k, b, p.total_k, p.Nk);
        const int nqt = (sq.len + 127) / 128;
        if (ii >= nqt) return;
        i = nqt - 1 - ii;
        lp = p;
        lp.Nq = sq.len;
        lp.Nk = sk.len;
        lp.nqt = nqt;
        lp.nkb = (sk.len + 127) / 128;
        lp.off = sk.len - sq.len;
        qrow0 = sq.start;
        krow0 = sk.start;
    } else {
        bh = static_cast<int>(blockIdx.x % static_cast<unsigned>(p.nbh));
        i = p.nqt - 1 - static_cast<int>(blockIdx.x / static_cast<unsigned>(p.nbh));
        plane = bh;
    }
    const BwdParams &ip = pick<VARLEN>(lp, p);

    auto bar = [&](int x) -> uint32_t { return sbase + C::kBarOff + 8u * x; };
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + C::kMiscOff);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::kMiscOff + 4);

    if (threadIdx.x == 0) {
        mbar_init(bar(C::kBarQ), 1);
        for (int s = 0; s < C::kKBars; ++s) {
            mbar_init(bar(C::kBarKFull + s), 1);
            mbar_init(bar(C::kBarKEmpty + s), 1);
        }
        for (int s = 0; s < NSV; ++s) {
            mbar_init(bar(C::kBarVFull + s), 1);
            mbar_init(bar(C::kBarVEmpty + s), 1);
        }
        for (int b = 0; b < NSB; ++b) {
            mbar_init(bar(C::kBarSFull + b), 1);
            mbar_init(bar(C::kBarDsFull + b), 256);
        }
        mbar_init(bar(C::kBarDPFull), 1);
        mbar_init(bar(C::kBarDPFree), 256);
        mbar_init(bar(C::kBarMmaDone), 1);
        *abort_flag = 0;
        mbar_fence_init();
    }
    if (warp == C::kWarpMma) {
        tmem_alloc(smem_u32(tmem_holder), 512);
        tmem_relinquish();
    }
    if (warp == C::kWarpTmaK && lane == 0) {
        tma_prefetch_desc(&tmq);
        tma_prefetch_desc(&tmk);
        tma_prefetch_desc(&tmv);
        tma_prefetch_desc(&tmdo);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    int cnt = 0;        // key blocks processed by this warp's role
    bool ok = true;

    if (warp == C::kWarpTmaK) {
        // ------------------------------------------------------------ Q, dO and K
        if (lane == 0) {
            mbar_arrive_expect_tx(bar(C::kBarQ), 2 * C::kTile);
            for (int c = 0; c < D / 64; ++c) {
                tma_load_3d(sbase + C::kQOff + c * C::kChunk, &tmq, bar(C::kBarQ), c * 64, qrow0 + i * 128, plane);
                tma_load_3d(sbase + C::kdOOff + c * C::kChunk, &tmdo, bar(C::kBarQ), c * 64, qrow0 + i * 128, plane);
            }
        }
        __syncwarp();
        KIter<GENERAL> it;
        int j;
        while (it.next(ip, i, j)) {
            if constexpr (C::kWide) {
                // two halves of K_j, each refilled once the dQ half that reads it is done
                for (int h = 0; h < 2 && ok; ++h) {
                    ok = wait_bar(bar(C::kBarKEmpty + h), (cnt & 1) ^ 1u, abort_flag);
                    if (!ok) break;
                    if (lane == 0) {
                        mbar_arrive_expect_tx(bar(C::kBarKFull + h), 2 * C::kChunk);
                        for (int c = 2 * h; c < 2 * h + 2; ++c)
                            tma_load_3d(sbase + C::kKOff + c * C::kChunk, &tmk, bar(C::kBarKFull + h), c * 64,
                                        krow0 + j * 128, plane);
                    }
                    __syncwarp();
                }
                if (!ok) break;
            } else {
                const int s = cnt % NSK;
                ok = wait_bar(bar(C::kBarKEmpty + s), ((cnt / NSK) & 1) ^ 1u, abort_flag);
                if (!ok) break;
                if (lane == 0) {
                    mbar_arrive_expect_tx(bar(C::kBarKFull + s), C::kTile);
                    for (int c = 0; c < D / 64; ++c)
                        tma_load_3d(sbase + C::kKOff + s * C::kTile + c * C::kChunk, &tmk, bar(C::kBarKFull + s),
                                    c * 64, krow0 + j * 128, plane);
                }
                __syncwarp();
            }
            ++cnt;
        }
        // every issued load has landed before the CTA may exit
        drain_bar(bar(C::kBarQ), 0);
        if constexpr (C::kWide) {
            if (cnt > 0)
                for (int h = 0; h < 2; ++h) drain_bar(bar(C::kBarKFull + h), (cnt - 1) & 1);
        } else {
            for (int x = (cnt > NSK ? cnt - NSK : 0); x < cnt; ++x) drain_bar(bar(C::kBarKFull + x % NSK), (x / NSK) & 1);
        }
    } else if (warp == C::kWarpTmaV) {
        // ------------------------------------------------------------ V
        constexpr int kLoadsPerBlock = C::kWide ? D / 64 : 1;
        KIter<GENERAL> it;
        int j;
        while (ok && it.next(ip, i, j)) {
            for (int u = 0; u < kLoadsPerBlock; ++u) {   // cnt counts V slots filled
                const int s = cnt % NSV;
                ok = wait_bar(bar(C::kBarVEmpty + s), ((cnt / NSV) & 1) ^ 1u, abort_flag);
                if (!ok) break;
                if (lane == 0) {
                    mbar_arrive_expect_tx(bar(C::kBarVFull + s), C::kVSlot);
                    if constexpr (C::kWide) {
                        tma_load_3d(sbase + C::kVOff + s * C::kVSlot, &tmv, bar(C::kBarVFull + s), u * 64,
                                    krow0 + j * 128, plane);
                    } else {
                        for (int c = 0; c < D / 64; ++c)
                            tma_load_3d(sbase + C::kVOff + s * C::kVSlot + c * C::kChunk, &tmv, bar(C::kBarVFull + s),
                                        c * 64, krow0 + j * 128, plane);
                    }
                }
                __syncwarp();
                ++cnt;
            }
        }
        for (int x = (cnt > NSV ? cnt - NSV : 0); x < cnt; ++x) drain_bar(bar(C::kBarVFull + x % NSV), (x / NSV) & 1);
    } else if (warp == C::kWarpMma) {
        // ------------------------------------------------------------ MMA issuer
        const uint32_t leader = elect_one();   // the lane that issues tcgen05 ops
        constexpr uint32_t kIdS = instr_desc_f16(128, 128, BF16, false, false);          // S, dP
        constexpr uint32_t kIdQ = instr_desc_f16(128, C::kWide ? 128 : D, BF16, false, true);   // dQ (a half at d = 256)
        // descriptors built once; each instruction only offsets the start address
        const SmemDesc dQ_k = make_desc(sbase + C::kQOff, 16, 1024);
        const SmemDesc ddO_k = make_desc(sbase + C::kdOOff, 16, 1024);
        const SmemDesc dK_k = make_desc(sbase + C::kKOff, 16, 1024);
        const SmemDesc dV_k = make_desc(sbase + C::kVOff, 16, 1024);
        const SmemDesc dK_mn = make_desc(sbase + C::kKOff, C::kChunk, 1024);
        // S = Q_i K_j^T over d indices [16 k0, 16 k1) (K tile at byte offset ko)
        auto issue_s = [&](int b, uint32_t ko, int k0, int k1) {
#pragma unroll
            for (int k = k0; k < k1; ++k) {
                const uint32_t o = (k >> 2) * C::kChunk + (k & 3) * 32;
                mma_ss(tmem + C::kColS + 128 * b, dQ_k.at(o), dK_k.at(ko + o), kIdS, k > 0 ? 1u : 0u, leader);
            }
        };
        // dP (+)= dO_i V_j^T over the d indices of one V slot holding d chunks [c0, c0 + D / 64 or 1)
        auto issue_dp = [&](int sv, int c0, bool acc) {
            constexpr int kSteps = C::kWide ? 4 : D / 16;
#pragma unroll
            for (int k = 0; k < kSteps; ++k) {
                const uint32_t ov = (k >> 2) * C::kChunk + (k & 3) * 32;
                const uint32_t oq = (c0 + (k >> 2)) * C::kChunk + (k & 3) * 32;
                mma_ss(tmem + C::kColDP, ddO_k.at(oq), dV_k.at(sv * C::kVSlot + ov), kIdS, (acc || k > 0) ? 1u : 0u,
                       leader);
            }
        };
        // dQ[:, cols] += dS K_j[:, cols]; dS of keys 16k.. at column 8k + 32 (k / 4) of the S buffer
        auto issue_dq = [&](int b, uint32_t ko, int col, bool acc) {
#pragma unroll
            for (int k = 0; k < 8; ++k)
                mma_ts(tmem + C::kColDQ + col, tmem + C::kColS + 128 * b + 8 * k + 32 * (k >> 2),
                       dK_mn.at(ko + k * 2048), kIdQ, (acc || k > 0) ? 1u : 0u, leader);
        };

        KIter<GENERAL> it;
        int jx;
        bool have = it.next(ip, i, jx);
        if constexpr (C::kWide) {
            int nv = 0;   // V chunks consumed
            auto full_s = [&](int c) -> bool {   // S(c) from the two K halves
                for (int h = 0; h < 2; ++h) {
                    if (!wait_bar(bar(C::kBarKFull + h), c & 1, abort_flag)) return false;
                    tc_fence_after();
                    issue_s(0, 0, 8 * h, 8 * h + 8);
                    __syncwarp();
                }
                mma_commit(bar(C::kBarSFull), leader);
                __syncwarp();
                return true;
            };
            auto full_dp = [&]() -> bool {        // dP(c) from four V chunks
                for (int u = 0; u < D / 64; ++u) {
                    const int s = nv % NSV;
                    if (!wait_bar(bar(C::kBarVFull + s), (nv / NSV) & 1, abort_flag)) return false;
                    tc_fence_after();
                    issue_dp(s, u, u > 0);
                    mma_commit(bar(C::kBarVEmpty + s), leader);
                    __syncwarp();
                    ++nv;
                }
                mma_commit(bar(C::kBarDPFull), leader);
                __syncwarp();
                return true;
            };
            if (have) {
                ok = wait_bar(bar(C::kBarQ), 0, abort_flag) && full_s(0) && full_dp();
            }
            while (ok && have) {
                const bool have_n = it.next(ip, i, jx);
                ok = wait_bar(bar(C::kBarDsFull), cnt & 1, abort_flag);
                if (!ok) break;
                tc_fence_after();
                for (int h = 0; h < 2; ++h) {
                    issue_dq(0, 2 * h * C::kChunk, 128 * h, cnt > 0);
                    mma_commit(bar(C::kBarKEmpty + h), leader);
                }
                __syncwarp();
                if (have_n) {
                    // dP(c + 1) overwrites dP(c): the softmax-grad warps have read it
                    ok = full_s(cnt + 1) && wait_bar(bar(C::kBarDPFree), cnt & 1, abort_flag) && full_dp();
                    if (!ok) break;
                }
                ++cnt;
                have = have_n;
            }
        } else {
            bool have_n = false;
            if (have) {
                have_n = it.next(ip, i, jx);
                ok = wait_bar(bar(C::kBarQ), 0, abort_flag) && wait_bar(bar(C::kBarKFull), 0, abort_flag) &&
                     wait_bar(bar(C::kBarVFull), 0, abort_flag);
                if (ok) {
                    tc_fence_after();
                    issue_s(0, 0, 0, D / 16);
                    mma_commit(bar(C::kBarSFull), leader);
                    issue_dp(0, 0, false);
                    mma_commit(bar(C::kBarDPFull), leader);
                    mma_commit(bar(C::kBarVEmpty), leader);
                    __syncwarp();
                }
                if (ok && have_n) {
                    ok = wait_bar(bar(C::kBarKFull + 1 % NSK), (1 / NSK) & 1, abort_flag);
                    if (ok) {
                        tc_fence_after();
                        issue_s(1, (1 % NSK) * C::kTile, 0, D / 16);
                        mma_commit(bar(C::kBarSFull + 1), leader);
                        __syncwarp();
                    }
                }
            }
            while (ok && have) {
                const int c = cnt;
                const bool have_nn = have_n && it.next(ip, i, jx);
                if (have_n) {
                    // dP(c + 1) once the softmax-grad warps have read dP(c)
                    const int sv = (c + 1) % NSV;
                    ok = wait_bar(bar(C::kBarDPFree), c & 1, abort_flag) &&
                         wait_bar(bar(C::kBarVFull + sv), ((c + 1) / NSV) & 1, abort_flag);
                    if (!ok) break;
                    tc_fence_after();
                    issue_dp(sv, 0, false);
                    mma_commit(bar(C::kBarDPFull), leader);
                    mma_commit(bar(C::kBarVEmpty + sv), leader);
                    __syncwarp();
                }
                ok = wait_bar(bar(C::kBarDsFull + (c & 1)), (c >> 1) & 1, abort_flag);
                if (!ok) break;
                tc_fence_after();
                issue_dq(c & 1, (c % NSK) * C::kTile, 0, c > 0);
                mma_commit(bar(C::kBarKEmpty + c % NSK), leader);
                __syncwarp();
                if (have_nn) {
                    const int sk = (c + 2) % NSK;
                    ok = wait_bar(bar(C::kBarKFull + sk), ((c + 2) / NSK) & 1, abort_flag);
                    if (!ok) break;
                    tc_fence_after();
                    issue_s(c & 1, sk * C::kTile, 0, D / 16);
                    mma_commit(bar(C::kBarSFull + (c & 1)), leader);
                    __syncwarp();
                }
                ++cnt;
                have = have_n;
                have_n = have_nn;
            }
        }
        mma_commit(bar(C::kBarMmaDone), leader);
        __syncwarp();
        drain_bar(bar(C::kBarMmaDone), 0);
    } else if (warp < 8) {
        // ------------------------------------------------------------ softmax-grad
        const int wq = warp & 3;
        const int kh = warp >> 2;             // key half of every block
        const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
        const int row = wq * 32 + lane;       // query row within the tile (TMEM lane)
        const int q = i * 128 + row;
        const size_t srow = static_cast<size_t>(bh) * p.Npad + q;   // q < nqt * 128 <= Npad
        const float l2 = p.lse2[srow];        // +inf past Nq or for rows that see no key: P = 0
        const float dd = p.dvec[srow];
        const float c2 = p.scale_log2;
        float sl = 0.f;
        if (GENERAL && p.alibi) sl = -p.alibi[bh % p.H] / p.scale;
        KIter<GENERAL> it;
        int j;
        while (it.next(ip, i, j)) {
            const int b = cnt % NSB;
            const uint32_t ph = (cnt / NSB) & 1;
            const uint32_t tS = tmem + lane_off + C::kColS + 128 * b + 64 * kh;
            ok = wait_bar(bar(C::kBarSFull + b), ph, abort_flag);
            if (!ok) break;
            tc_fence_after();
            // keys kb0 + kk this row sees: lo <= kk <= hi (key q + off - wl ..
            // q + off + wr, below Nk); causal squares have off = 0, wr = 0
            const int kb0 = j * 128 + 64 * kh;
            const int rk = q + ip.off - kb0;   // |values| < 2^30 (Nq, Nk <= 2^28)
            const int lo = max(rk - p.wl, -1);
            const int hi = min(min(rk + p.wr, ip.Nk - 1 - kb0), 64);
            float pv[64];
            {
                uint32_t sr[64];
                tmem_ld32(tS, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
                tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
                tmem_wait_ld(sr);
                if (GENERAL && p.alibi) {
                    // score + bias / scale, bias = -slope |q + off - key|
                    const float base = static_cast<float>(rk);
#pragma unroll
                    for (int kk = 0; kk < 64; ++kk)
                        sr[kk] = __float_as_uint(fmaf(sl, fabsf(base - static_cast<float>(kk)), __uint_as_float(sr[kk])));
                }
#pragma unroll
                for (int kk = 0; kk < 64; ++kk) pv[kk] = ex2(fmaf(__uint_as_float(sr[kk]), c2, -l2));
            }
            if (__any_sync(0xffffffffu, lo > 0 || hi < 63)) {
#pragma unroll
                for (int kk = 0; kk < 64; ++kk)
                    if (kk < lo || kk > hi) pv[kk] = 0.f;
            }
            ok = wait_bar(bar(C::kBarDPFull), cnt & 1, abort_flag);
            if (!ok) break;
            tc_fence_after();
            // dS = P o (dP - D), rounded to 16 bits, packed over the first 32 of
            // this thread's 64 S columns (keys 2k, 2k + 1 in column k)
            uint32_t ds[32];
            {
                uint32_t pr[32];
                const uint32_t tP = tmem + lane_off + C::kColDP + 64 * kh;
                tmem_ld32(tP, pr);
                tmem_wait_ld(pr);
#pragma unroll
                for (int k = 0; k < 16; ++k)
                    ds[k] = pack2<BF16>(pv[2 * k] * (__uint_as_float(pr[2 * k]) - dd),
                                        pv[2 * k + 1] * (__uint_as_float(pr[2 * k + 1]) - dd));
                tmem_ld32(tP + 32, pr);
                tmem_wait_ld(pr);
                tc_fence_before();
                mbar_arrive(bar(C::kBarDPFree));
#pragma unroll
                for (int k = 0; k < 16; ++k)
                    ds[16 + k] = pack2<BF16>(pv[32 + 2 * k] * (__uint_as_float(pr[2 * k]) - dd),
                                             pv[33 + 2 * k] * (__uint_as_float(pr[2 * k + 1]) - dd));
            }
            tmem_st32(tS, ds);
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(bar(C::kBarDsFull + b));
            ++cnt;
        }
        // ------------------------------------------------------------ dQ epilogue
        // staged as 128-byte-swizzled 64-column chunks in the Q_i buffer (free
        // once every product has completed), written by TMA stores
        bool done = ok;
        if (done && cnt > 0) done = wait_bar(bar(C::kBarMmaDone), 0, abort_flag);
        tc_fence_after();
        // a tile that sees no key block never waited for its Q/dO loads: they
        // must land before the staging area (the Q buffer) is written
        if (done && cnt == 0) drain_bar(bar(C::kBarQ), 0);
        // packed batches: a tile that ends inside the next sequence's rows is
        // written row by row with plain stores (a TMA store clips only at the
        // end of the tensor)
        const int qrows = VARLEN ? ip.Nq - i * 128 : 128;
        if (done) {
            // this thread: row `row`, d columns [kh D / 2, (kh + 1) D / 2)
#pragma unroll 1
            for (int ch = 0; ch < D / 64; ++ch) {
                uint32_t v[32];
                if (cnt > 0) {
                    tmem_ld32_wait(tmem + lane_off + C::kColDQ + kh * (D / 2) + 32 * ch, v);
                } else {
#pragma unroll
                    for (int k = 0; k < 32; ++k) v[k] = 0u;   // a tile that sees no key: dQ = 0
                }
                uint32_t pk[16];
#pragma unroll
                for (int k = 0; k < 16; ++k)
                    pk[k] = pack2<BF16>(__uint_as_float(v[2 * k]) * p.scale, __uint_as_float(v[2 * k + 1]) * p.scale);
                const int col = kh * (D / 2) + 32 * ch;
                if (VARLEN && qrows < 128) {
                    if (row < qrows) {
                        uint4 *g = reinterpret_cast<uint4 *>(
                            static_cast<uint8_t *>(p.dq) +
                            (static_cast<size_t>(qrow0 + i * 128 + row) * p.H + plane) * (D * 2) + col * 2);
#pragma unroll
                        for (int k = 0; k < 4; ++k)
                            g[k] = make_uint4(pk[4 * k], pk[4 * k + 1], pk[4 * k + 2], pk[4 * k + 3]);
                    }
                    continue;
                }
                uint8_t *srow = smem + C::kQOff + (col / 64) * C::kChunk + row * 128;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int u = (col % 64) / 8 + k;
                    *reinterpret_cast<uint4 *>(srow + ((u ^ (row & 7)) << 4)) =
                        make_uint4(pk[4 * k], pk[4 * k + 1], pk[4 * k + 2], pk[4 * k + 3]);
                }
            }
        }
        fence_async_smem();
        named_sync(1, 256);   // the eight softmax-grad warps (every one gets here)
        if (done && qrows >= 128 && warp == 0 && lane == 0) {
            for (int c = 0; c < D / 64; ++c)   // rows >= Nq are clipped
                tma_store_3d(&tmdq, smem_u32(smem + C::kQOff + c * C::kChunk), c * 64, qrow0 + i * 128, plane);
            bulk_commit();
            bulk_wait_read();
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == C::kWarpMma) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace fa
