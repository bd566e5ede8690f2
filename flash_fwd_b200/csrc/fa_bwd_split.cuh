// fa_bwd_split.cuh -- backward main kernel for d = 256 on sm_100a.
//
// The accumulators dK, dV of one 128-key block at d = 256 need 512 TMEM
// columns on their own, so the output columns are split over DSPLIT = 2 CTAs
// per key block: each CTA recomputes S^T and dP^T over the full d (two of the
// five products twice) and owns half of the dK, dV and dQ columns.  Query
// tiles have BM = 64 rows and one Q/dO stage fits shared memory; dQ^T =
// K_j^T dS^T (M = 128 output columns) is drained with fp32 atomics.
// The d <= 128 kernel (fa_bwd.cuh) describes the products and warp roles.
#pragma once

#include "fa_bwd.cuh"

namespace fa {

template <int D, int BM, int DSPLIT, int NS, int NPB, bool DQT>
struct BwdSplitCfg {
    static constexpr int DH = D / DSPLIT;                 // output columns per CTA
    static constexpr int kKVTile = 128 * D * 2;           // K_j or V_j
    static constexpr int kKVChunk = 128 * 128;            // 64 columns of a 128-row tile
    static constexpr int kQTile = BM * D * 2;             // Q_i or dO_i
    static constexpr int kQChunk = BM * 128;              // 64 columns of a BM-row tile
    static constexpr int kPTile = 128 * BM * 2;           // P^T or dS^T: 128 keys x BM queries
    static constexpr int kKOff = 0;
    static constexpr int kVOff = kKOff + kKVTile;
    static constexpr int kQOff = kVOff + kKVTile;
    static constexpr int kdOOff = kQOff + NS * kQTile;
    static constexpr int kdSOff = kdOOff + NS * kQTile;   // NPB buffers of dS^T
    static constexpr int kStatOff = kdSOff + NPB * kPTile;   // per stage: lse*log2e [BM], D [BM]
    static constexpr int kBarOff = kStatOff + NS * BM * 8;
    static constexpr int kBarKV = 0;
    static constexpr int kBarQFull = 1;
    static constexpr int kBarQEmpty = kBarQFull + NS;
    static constexpr int kBarSdpFull = kBarQEmpty + NS;
    static constexpr int kBarSdpEmpty = kBarSdpFull + 1;
    static constexpr int kBarDsFull = kBarSdpEmpty + 1;
    static constexpr int kBarPdsEmpty = kBarDsFull + 1;   // NPB barriers, one per P/dS buffer
    static constexpr int kBarDqFull = kBarPdsEmpty + NPB;
    static constexpr int kBarDqEmpty = kBarDqFull + 1;
    static constexpr int kBarMmaDone = kBarDqEmpty + 1;
    static constexpr int kNumBars = kBarMmaDone + 1;
    static constexpr int kMiscOff = kBarOff + kNumBars * 8;
    static constexpr int kSmemBytes = kMiscOff + 16 + 1024;
    static constexpr int kThreads = 320;
    static constexpr int kColS = 0;
    static constexpr int kColDP = 128;
    static constexpr int kColDV = 256;
    static constexpr int kColDK = 256 + DH;
    static constexpr int kColDQ = DQT ? 64 : 256 + 2 * DH;
    static constexpr int kDqCols = DQT ? BM : DH;         // fp32 columns per drain thread
    static constexpr int kColPT = DQT ? 192 : 448;        // NPB buffers of 16-bit P^T (BM / 2 columns each)
    static constexpr int kStatBytes = BM * 4;
    // CTA order: heads in groups of kHeadGroup, key-block columns major within
    // a group (heaviest first under causal), heads minor; the running CTAs then
    // reduce into the fp32 dQ rows of kHeadGroup heads only (at d = 256 the
    // accumulator of all heads is far larger than L2).  Measured at B=4 H=16
    // N=4096 causal: 3.99 ms per launch with one group of all 64 heads, 3.70
    // with groups of 4 or 8, 3.75 with 16
    static constexpr int kHeadGroup = 8;
    static_assert(kColPT + NPB * BM / 2 <= (DQT ? 256 : 512), "P^T columns");
    static_assert(DQT ? (BM == 64 && DH == 128) : (BM == 128 && DH == 64), "tile shape");
    static_assert(kColDQ + kDqCols <= 512 && kColDK + DH <= 512, "TMEM columns");
    static_assert(NPB == 1 || NPB == 2, "P/dS buffers");
    static_assert(kSmemBytes <= 227 * 1024, "shared memory");
};

template <int D, int BM, int DSPLIT, int NS, int NPB, bool DQT, bool BF16, bool GENERAL, bool VARLEN = false>
__global__ void __launch_bounds__(320, 1)
    bwd_split_kernel(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
               const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmdo,
               const __grid_constant__ CUtensorMap tmdk, const __grid_constant__ CUtensorMap tmdv,
               const BwdParams p) {
    using C = BwdSplitCfg<D, BM, DSPLIT, NS, NPB, DQT>;
    constexpr int DH = C::DH;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = smem_u32(smem);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    static_assert(GENERAL || !VARLEN, "packed batches use the general band");
    // one-dimensional grid: groups of kHeadGroup heads, (batch, head) minor
    // within a group (see bwd_kernel).  Packed batches: sequence major, then
    // (key block, column half), heads minor; a CTA past its own sequence's
    // keys leaves before any setup.
    int bh, jh;
    if constexpr (VARLEN) {
        const long long per = static_cast<long long>(p.H) * p.nkb * DSPLIT;
        const int b = static_cast<int>(blockIdx.x / per);
        const int r = static_cast<int>(blockIdx.x - b * per);
        jh = r / p.H;
        bh = b * p.H + (r - jh * p.H);
    } else {
        const int hg = min(C::kHeadGroup, p.nbh);
        const long long per = static_cast<long long>(hg) * p.nkb * DSPLIT;
        const int g = static_cast<int>(blockIdx.x / per);
        const int r = static_cast<int>(blockIdx.x - g * per);
        const int gh = min(hg, p.nbh - g * hg);   // heads in this group
        jh = r / gh;
        bh = g * hg + (r - jh * gh);
    }
    const int j = jh / DSPLIT;
    const int h = jh % DSPLIT;
    // packed batches: lp is p with this sequence's lengths; TMA rows are
    // offset by qrow0 / krow0 in plane (the head)
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

    auto bar = [&](int i) -> uint32_t { return sbase + C::kBarOff + 8u * i; };
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + C::kMiscOff);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::kMiscOff + 4);

    if (threadIdx.x == 0) {
        mbar_init(bar(C::kBarKV), 1);
        for (int s = 0; s < NS; ++s) {
            mbar_init(bar(C::kBarQFull + s), 1);
            mbar_init(bar(C::kBarQEmpty + s), 1);
        }
        mbar_init(bar(C::kBarSdpFull), 1);
        mbar_init(bar(C::kBarSdpEmpty), 128);
        mbar_init(bar(C::kBarDsFull), 128);
        for (int b = 0; b < NPB; ++b) mbar_init(bar(C::kBarPdsEmpty + b), 1);
        mbar_init(bar(C::kBarDqFull), 1);
        mbar_init(bar(C::kBarDqEmpty), 128);
        mbar_init(bar(C::kBarMmaDone), 1);
        *abort_flag = 0;
        mbar_fence_init();
    }
    if (warp == 9) {
        tmem_alloc(smem_u32(tmem_holder), 512);
        tmem_relinquish();
    }
    if (warp == 8 && lane == 0) {
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

    if (warp == 8) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            mbar_arrive_expect_tx(bar(C::kBarKV), 2 * C::kKVTile);
            for (int c = 0; c < D / 64; ++c) {
                tma_load_3d(sbase + C::kKOff + c * C::kKVChunk, &tmk, bar(C::kBarKV), c * 64, krow0 + j * 128,
                            plane);
                tma_load_3d(sbase + C::kVOff + c * C::kKVChunk, &tmv, bar(C::kBarKV), c * 64, krow0 + j * 128,
                            plane);
            }
        }
        __syncwarp();
        QIter<BM, GENERAL> it;
        int i;
        while (it.next(ip, j, i)) {
            const int s = cnt % NS;
            const uint32_t ph = (cnt / NS) & 1;
            ok = wait_bar(bar(C::kBarQEmpty + s), ph ^ 1u, abort_flag);
            if (!ok) break;
            // Q_i, dO_i (TMA tiles) and the padded per-row statistics (bulk
            // copies, prepared by bwd_pre) land on one transaction barrier
            if (lane == 0) {
                const uint32_t qb = bar(C::kBarQFull + s);
                mbar_arrive_expect_tx(qb, 2 * C::kQTile + 2 * C::kStatBytes);
                for (int c = 0; c < D / 64; ++c) {
                    tma_load_3d(sbase + C::kQOff + s * C::kQTile + c * C::kQChunk, &tmq, qb, c * 64,
                                qrow0 + i * BM, plane);
                    tma_load_3d(sbase + C::kdOOff + s * C::kQTile + c * C::kQChunk, &tmdo, qb, c * 64,
                                qrow0 + i * BM, plane);
                }
                const size_t srow = static_cast<size_t>(bh) * p.Npad + static_cast<size_t>(i) * BM;
                bulk_load(sbase + C::kStatOff + s * 2 * C::kStatBytes, p.lse2 + srow, C::kStatBytes, qb);
                bulk_load(sbase + C::kStatOff + s * 2 * C::kStatBytes + C::kStatBytes, p.dvec + srow,
                          C::kStatBytes, qb);
            }
            __syncwarp();
            ++cnt;
        }
        drain_bar(bar(C::kBarKV), 0);
        for (int x = (cnt > NS ? cnt - NS : 0); x < cnt; ++x) drain_bar(bar(C::kBarQFull + x % NS), (x / NS) & 1);
    } else if (warp == 9) {
        // ------------------------------------------------------------ MMA issuer
        const uint32_t leader = elect_one();   // the lane that issues tcgen05 ops
        constexpr uint32_t kIdS = instr_desc_f16(128, BM, BF16, false, false);
        constexpr uint32_t kIdKV = instr_desc_f16(128, DH, BF16, false, true);
        constexpr uint32_t kIdQ = DQT ? instr_desc_f16(128, BM, BF16, true, true)
                                      : instr_desc_f16(128, DH, BF16, true, true);
        // descriptors built once; each instruction only offsets the start address
        const SmemDesc dK_kmaj = make_desc(sbase + C::kKOff, 16, 1024);
        const SmemDesc dV_kmaj = make_desc(sbase + C::kVOff, 16, 1024);
        const SmemDesc dQ_kmaj = make_desc(sbase + C::kQOff, 16, 1024);
        const SmemDesc ddO_kmaj = make_desc(sbase + C::kdOOff, 16, 1024);
        const SmemDesc dQ_mn = make_desc(sbase + C::kQOff + h * (DH / 64) * C::kQChunk, C::kQChunk, 1024);
        const SmemDesc ddO_mn = make_desc(sbase + C::kdOOff + h * (DH / 64) * C::kQChunk, C::kQChunk, 1024);
        const SmemDesc ddS_kmaj = make_desc(sbase + C::kdSOff, 16, 1024);
        const SmemDesc ddS_mn = make_desc(sbase + C::kdSOff, 128 * 128, 1024);
        const SmemDesc dK_mn = make_desc(sbase + C::kKOff + h * (DH / 64) * C::kKVChunk, C::kKVChunk, 1024);
        auto issue_sdp = [&](int s) {
#pragma unroll
            for (int k = 0; k < D / 16; ++k) {
                const uint32_t okv = (k >> 2) * C::kKVChunk + (k & 3) * 32;
                const uint32_t oq = s * C::kQTile + (k >> 2) * C::kQChunk + (k & 3) * 32;
                mma_ss(tmem + C::kColS, dK_kmaj.at(okv), dQ_kmaj.at(oq), kIdS, k > 0 ? 1u : 0u, leader);
            }
#pragma unroll
            for (int k = 0; k < D / 16; ++k) {
                const uint32_t okv = (k >> 2) * C::kKVChunk + (k & 3) * 32;
                const uint32_t oq = s * C::kQTile + (k >> 2) * C::kQChunk + (k & 3) * 32;
                mma_ss(tmem + C::kColDP, dV_kmaj.at(okv), ddO_kmaj.at(oq), kIdS, k > 0 ? 1u : 0u, leader);
            }
        };
        auto issue_dvdk = [&](int s, int pb, bool acc) {
#pragma unroll
            for (int k = 0; k < BM / 16; ++k)   // dV += P^T dO_i, P^T read from TMEM
                mma_ts(tmem + C::kColDV, tmem + C::kColPT + pb * (BM / 2) + 8 * k,
                       ddO_mn.at(s * C::kQTile + k * 2048), kIdKV, (acc || k > 0) ? 1u : 0u, leader);
#pragma unroll
            for (int k = 0; k < BM / 16; ++k) {
                const uint32_t oa = pb * C::kPTile + (k >> 2) * (128 * 128) + (k & 3) * 32;
                mma_ss(tmem + C::kColDK, ddS_kmaj.at(oa), dQ_mn.at(s * C::kQTile + k * 2048), kIdKV,
                       (acc || k > 0) ? 1u : 0u, leader);
            }
        };
        auto issue_dq = [&](int pb) {
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                if constexpr (DQT) {
                    // dQ^T (DH x BM) = K_j^T (DH x 128 keys) * dS^T (128 keys x BM)
                    mma_ss(tmem + C::kColDQ, dK_mn.at(k * 2048), ddS_mn.at(pb * C::kPTile + k * 2048), kIdQ,
                           k > 0 ? 1u : 0u, leader);
                } else {
                    // dQ (BM x DH) = dS (BM x 128 keys) * K_j (128 keys x DH)
                    mma_ss(tmem + C::kColDQ, ddS_mn.at(pb * C::kPTile + k * 2048), dK_mn.at(k * 2048), kIdQ,
                           k > 0 ? 1u : 0u, leader);
                }
            }
        };

        QIter<BM, GENERAL> it;
        int i, in;
        bool have = it.next(ip, j, i);
        if (have) {
            ok = wait_bar(bar(C::kBarKV), 0, abort_flag) && wait_bar(bar(C::kBarQFull), 0, abort_flag);
            if (ok) {
                tc_fence_after();
                {
                    issue_sdp(0);
                    mma_commit(bar(C::kBarSdpFull), leader);
                }
                __syncwarp();
            }
        }
        // S^T, dP^T of the next tile: needs the softmax-grad warps to have read
        // this tile's and the producer to have landed the next Q_i, dO_i
        auto prefetch_next = [&]() -> bool {
            const int sn = (cnt + 1) % NS;
            if (!(wait_bar(bar(C::kBarSdpEmpty), cnt & 1, abort_flag) &&
                  wait_bar(bar(C::kBarQFull + sn), ((cnt + 1) / NS) & 1, abort_flag)))
                return false;
            tc_fence_after();
            {
                issue_sdp(sn);
                mma_commit(bar(C::kBarSdpFull), leader);
            }
            __syncwarp();
            return true;
        };
        while (ok && have) {
            const int s = cnt % NS;
            const int pb = cnt % NPB;
            const bool have_n = it.next(ip, j, in);
            // with two or more stages the next tile is already resident: overlap
            // its S^T, dP^T with this tile's softmax-grad work.  With one stage
            // the next tile can only land after this tile's products finish.
            if (NS >= 2 && have_n) {
                ok = prefetch_next();
                if (!ok) break;
            }
            ok = wait_bar(bar(C::kBarDsFull), cnt & 1, abort_flag);
            if (!ok) break;
            tc_fence_after();
            issue_dvdk(s, pb, cnt > 0);
            __syncwarp();
            const bool with_dq = p.dqacc != nullptr;   // else the deterministic dQ pass computes dQ
            ok = !with_dq || wait_bar(bar(C::kBarDqEmpty), (cnt & 1) ^ 1u, abort_flag);
            if (!ok) break;
            tc_fence_after();
            {
                if (with_dq) {
                    issue_dq(pb);
                    mma_commit(bar(C::kBarDqFull), leader);
                }
                mma_commit(bar(C::kBarPdsEmpty + pb), leader);
                mma_commit(bar(C::kBarQEmpty + s), leader);
            }
            __syncwarp();
            if (NS == 1 && have_n) {
                ok = prefetch_next();
                if (!ok) break;
            }
            ++cnt;
            have = have_n;
            i = in;
        }
        mma_commit(bar(C::kBarMmaDone), leader);
        __syncwarp();
        drain_bar(bar(C::kBarMmaDone), 0);
    } else if (warp < 4) {
        // ------------------------------------------------------------ softmax-grad
        const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
        const int r = warp * 32 + lane;     // key row within the block
        const int key = j * 128 + r;
        const float c = p.scale_log2;
        QIter<BM, GENERAL> it;
        int i;
        while (it.next(ip, j, i)) {
            const int s = cnt % NS;
            const int pb = cnt % NPB;
            uint8_t *sdS = smem + C::kdSOff + pb * C::kPTile;
            const uint32_t tP = tmem + lane_off + C::kColPT + pb * (BM / 2);
            ok = wait_bar(bar(C::kBarSdpFull), cnt & 1, abort_flag) &&
                 wait_bar(bar(C::kBarQFull + s), (cnt / NS) & 1, abort_flag);
            if (!ok) break;
            tc_fence_after();
            const float4 *lse4 = reinterpret_cast<const float4 *>(smem + C::kStatOff + s * 2 * C::kStatBytes);
            const float4 *dd4 = lse4 + BM / 4;
            // queries i * BM + kk that see key `key`: lo <= kk <= hi (key q + off - wl ..
            // q + off + wr); keys past Nk see none
            int qk, lo, hi;
            bool masked;
            if constexpr (GENERAL) {
                qk = key - ip.off - i * BM;     // |values| < 2^30 (Nq, Nk <= 2^28)
                lo = max(qk - p.wr, -1);
                hi = min(qk + p.wl, BM);
                if (key >= ip.Nk) lo = BM;
                masked = __any_sync(0xffffffffu, lo > 0 || hi < BM - 1);
            } else {
                // square: queries before the key are hidden on the diagonal tiles
                qk = 0;
                hi = BM;
                lo = key - i * BM;
                masked = (p.mode & kCausal) && (i * BM < j * 128 + 127);
            }
#pragma unroll 1
            for (int ch = 0; ch < BM / 32; ++ch) {
                uint32_t sr[32], pr[32];
                tmem_ld32(tmem + lane_off + C::kColS + 32 * ch, sr);
                tmem_ld32(tmem + lane_off + C::kColDP + 32 * ch, pr);
                tmem_wait_ld(sr, pr);
                if (GENERAL && p.alibi) {
                    // score + bias / scale, bias = -slope |q + off - key|
                    const float sl = -p.alibi[bh % p.H] / p.scale;
                    const float base = static_cast<float>(-qk + 32 * ch);
#pragma unroll
                    for (int kk = 0; kk < 32; ++kk)
                        sr[kk] = __float_as_uint(fmaf(sl, fabsf(base + static_cast<float>(kk)), __uint_as_float(sr[kk])));
                }
                if (ch == BM / 32 - 1) {
                    tc_fence_before();
                    mbar_arrive(bar(C::kBarSdpEmpty));
                }
                uint32_t pk[16], dk[16];
#pragma unroll
                for (int k4 = 0; k4 < 8; ++k4) {
                    const float4 l4 = lse4[ch * 8 + k4];
                    const float4 d4 = dd4[ch * 8 + k4];
                    const float lv[4] = {l4.x, l4.y, l4.z, l4.w};
                    const float dv[4] = {d4.x, d4.y, d4.z, d4.w};
                    float pp[4], ds[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int kk = 4 * k4 + e;
                        float pv = ex2(fmaf(__uint_as_float(sr[kk]), c, -lv[e]));
                        if (masked && (32 * ch + kk < lo || 32 * ch + kk > hi)) pv = 0.f;
                        pp[e] = pv;
                        ds[e] = pv * (__uint_as_float(pr[kk]) - dv[e]);
                    }
                    pk[2 * k4] = pack2<BF16>(pp[0], pp[1]);
                    pk[2 * k4 + 1] = pack2<BF16>(pp[2], pp[3]);
                    dk[2 * k4] = pack2<BF16>(ds[0], ds[1]);
                    dk[2 * k4 + 1] = pack2<BF16>(ds[2], ds[3]);
                }
                if (ch == 0 && cnt >= NPB) {
                    // the products that read this P/dS buffer NPB tiles ago must be done
                    if (!wait_bar(bar(C::kBarPdsEmpty + pb), ((cnt / NPB) - 1) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                }
                // P^T row r -> TMEM (A operand of dV); dS^T row r -> a K-major
                // [BM/64][128][64] 128B-swizzled shared tile (dK and dQ operand)
                tmem_st16(tP + 16 * ch, pk);
                const int chunk = (32 * ch) / 64;
                const int u0 = ((32 * ch) % 64) / 8;
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int off = chunk * (128 * 128) + r * 128 + (((u0 + u) ^ (r & 7)) << 4);
                    *reinterpret_cast<uint4 *>(sdS + off) = make_uint4(dk[4 * u], dk[4 * u + 1], dk[4 * u + 2], dk[4 * u + 3]);
                }
            }
            if (!ok) break;
            tmem_st_wait();
            tc_fence_before();
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            mbar_arrive(bar(C::kBarDsFull));
            ++cnt;
        }
    } else {
        // ------------------------------------------------------------ dQ drain
        const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const int t = (warp & 3) * 32 + lane;   // TMEM lane: a d index (transposed form) or a query row
        QIter<BM, GENERAL> it;
        int i;
        while (it.next(ip, j, i)) {
            if (p.dqacc == nullptr) {   // no dQ: only count the tiles (the dK epilogue needs cnt)
                ++cnt;
                continue;
            }
            ok = wait_bar(bar(C::kBarDqFull), cnt & 1, abort_flag);
            if (!ok) break;
            tc_fence_after();
            uint32_t v[C::kDqCols];
            if constexpr (C::kDqCols == 64) tmem_ld64_wait(tmem + lane_off + C::kColDQ, v);
            else tmem_ld128_wait(tmem + lane_off + C::kColDQ, v);
            tc_fence_before();
            mbar_arrive(bar(C::kBarDqEmpty));
            // accumulator rows of this (b, h): [BH][Nq][D], packed batches [H][total_q][D]
            float *accb = p.dqacc + (VARLEN ? static_cast<size_t>(plane) * p.total_q + qrow0
                                            : static_cast<size_t>(bh) * p.Nq) * D;
            if constexpr (DQT) {
                const int dcol = h * DH + t;
#pragma unroll
                for (int k = 0; k < BM; ++k) {
                    const int q = i * BM + k;
                    if (q < ip.Nq) atomicAdd(accb + static_cast<size_t>(q) * D + dcol, __uint_as_float(v[k]));
                }
            } else {
                const int q = i * BM + t;
                if (q < ip.Nq) {
                    float4 *dst = reinterpret_cast<float4 *>(accb + static_cast<size_t>(q) * D + h * DH);
#pragma unroll
                    for (int k = 0; k < DH / 4; ++k)
                        atomicAdd(dst + k, make_float4(__uint_as_float(v[4 * k]), __uint_as_float(v[4 * k + 1]),
                                                       __uint_as_float(v[4 * k + 2]), __uint_as_float(v[4 * k + 3])));
                }
            }
            ++cnt;
        }
    }

    // ---------------------------------------------------------------- dV / dK epilogue
    if (warp < 8) {
        // this CTA's DH columns of dV (warps 0-3) / dK (warps 4-7), staged as
        // 128-byte-swizzled 64-column chunks in the V_j / K_j buffers (free once
        // every product has completed) and written by TMA stores
        bool done = ok;
        if (done && cnt > 0) done = wait_bar(bar(C::kBarMmaDone), 0, abort_flag);
        tc_fence_after();
        const bool is_dv = warp < 4;
        const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const int r = (warp & 3) * 32 + lane;
        const float mul = is_dv ? 1.0f : p.scale;
        uint8_t *stage = smem + (is_dv ? C::kVOff : C::kKOff);
        const uint32_t col0 = is_dv ? C::kColDV : C::kColDK;
        // a key block that no query tile sees never waited for its K/V loads:
        // they must land before the staging areas are written
        if (done && cnt == 0) drain_bar(bar(C::kBarKV), 0);
        // packed batches: a key block that ends inside the next sequence's
        // rows is written row by row with plain stores (a TMA store clips only
        // at the end of the tensor)
        const int krows = VARLEN ? ip.Nk - j * 128 : 128;
        if (done) {
#pragma unroll 1
            for (int ch = 0; ch < DH / 32; ++ch) {
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
                            (static_cast<size_t>(krow0 + j * 128 + r) * p.H + plane) * (D * 2) + (h * DH + ch * 32) * 2);
#pragma unroll
                        for (int k = 0; k < 4; ++k)
                            g[k] = make_uint4(pk[4 * k], pk[4 * k + 1], pk[4 * k + 2], pk[4 * k + 3]);
                    }
                    continue;
                }
                uint8_t *srow = stage + (ch >> 1) * C::kKVChunk + r * 128;
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
            for (int c = 0; c < DH / 64; ++c)   // keys >= Nk are clipped
                tma_store_3d(is_dv ? &tmdv : &tmdk, smem_u32(stage + c * C::kKVChunk), h * DH + c * 64,
                             krow0 + j * 128, plane);
            bulk_commit();
            bulk_wait_read();
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 9) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace fa
