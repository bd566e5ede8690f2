// fa_fwd.cuh -- forward kernel of exact attention for sm_100a.
//
// What it computes: for every (batch, head) and query row i,
//   O_i = sum_j softmax_j(scale * q_i . k_j) v_j,  LSE_i = ln sum_j exp(scale * q_i . k_j)
// over the keys visible to i, with the online softmax of "FlashAttention
// 深度解析" section 二: a running max m and sum l are corrected by
// 2^(m_old - m_new) whenever a key tile raises the max, O stays unnormalised
// and is divided by l once at the end (深度解析 section 四, deferred
// normalisation).  S and P live only in tensor memory ("FlashAttention原理概览"
// section 3.1: the intermediate S_ij and P_ij never reach device memory).
//
// Decomposition (the outer-Q / inner-K/V order of 深度解析 section 四): a
// work item is NQ query tiles of 128 rows of one (batch, head); the kept
// 128-key tiles of K and V stream through shared-memory rings of NSK (K) and
// NSV (V) stages.  With NQ = 2 the grid is one CTA per SM and each CTA runs
// its share of the items in turn (fwd_kernel describes the hand-over between
// items); with NQ = 1 (d = 256) every item is its own CTA.  K gets the deeper ring: S of the next key tile is issued
// right after P V of the current one, so its K tile is needed a whole
// softmax phase before its V tile.
//
// Warp roles (a B200 design; the pages' own schedules target A100/H100):
//   warps 0 .. 4*NQ-1   softmax: warpgroup t owns query tile t, one thread per
//                       row.  It reads S_t from TMEM, masks, updates m and l,
//                       rescales O_t in TMEM when m grew by more than 2^8
//                       (exactness is kept because O and l share the stale m),
//                       writes P_t (16-bit) back over S_t and signals the MMA
//                       warp once per half (keys 0..63, 64..127): O_t += P_t V
//                       starts on the first half while the second is computed.
//   warp 4*NQ           TMA producer: the item's Q tiles, then K_j per stage
//                       (and V_j when NQ = 1).
//   warp 4*NQ+2         (NQ = 2) TMA producer of the V_j tiles; it also issues
//                       the TMA stores of each item's O (staged in V stages
//                       0 .. NQ-1 by the softmax warps).
//   warp 4*NQ+1         MMA issuer (one elected lane): S_t = Q_t K_j^T (SS form)
//                       and O_t += P_t V_j (P read from TMEM, TS form).  It owns
//                       the 512-column TMEM allocation.
// TMEM columns: S_t at [128 t, 128 t + 128) (P_t reuses its first 64 columns),
// O_t at [256 + D t, 256 + D t + D).
//
// Scale handling: exp is evaluated as 2^(s * scale * log2 e - m), with the
// running max m kept in that base-2 domain; LSE converts back to natural log.
// exp2 runs on the special-function unit (16 results per clock per SM); a
// degree-3 polynomial on the FMA pipe (128 per clock) can take a share of
// the pairs (kPolyPairs); it is off (see the softmax loop for the measurements).
#pragma once

#include "fa_common.cuh"

namespace fa {

enum MaskMode : int { kDense = 0, kCausal = 1, kSparse = 2 };

struct FwdParams {
    float *lse;               // [BH][Nq]
    const uint8_t *mask;      // [nqb][nkb] block mask (kSparse)
    const float *alibi;       // [H] ALiBi slopes (natural-log units of the score) or null (GENERAL kernels)
    int Nq, Nk;               // query rows and keys per (b, h)
    int off, wl, wr;          // visibility band (see band_any)
    int nqb;                  // query blocks of 128 rows
    int nkb;                  // key blocks of 128 keys
    int nbh;                  // batch x heads
    int nitems;               // work items: nbh x ceil(nqb / NQ) query-tile groups
    int H;                    // heads (head of batch-head bh: bh % H)
    int mode;                 // kCausal (heaviest-first order) | kSparse bits
    float scale;
    float scale_log2;         // scale * log2(e)
    // packed variable-length batches (VARLEN kernels): sequence b owns packed
    // rows cu_q[b] .. cu_q[b+1]-1 of q and o and cu_k[b] .. cu_k[b+1]-1 of k
    // and v, each [rows][H][d]; lse is [H][total_q].  Nq, Nk, nqb and nkb
    // above then describe the longest sequences (they size the item grid).
    const int *cu_q;
    const int *cu_k;
    void *o;                  // packed O: the rows of a sequence's last, partial tile
    int total_q, total_k;     // packed rows
};

// Is key block j visible at all from query block rb?  GENERAL kernels handle
// Nq != Nk, windows and ALiBi through the visibility band; the others serve
// square problems (dense, causal, block-sparse) with the plain causal test.
template <bool GENERAL>
__device__ __forceinline__ bool block_kept(const FwdParams &p, int rb, int j) {
    if (rb >= p.nqb || j >= p.nkb) return false;
    if constexpr (GENERAL) {
        const int q0 = rb * 128, k0 = j * 128;
        const int q1 = min(q0 + 127, p.Nq - 1), k1 = min(k0 + 127, p.Nk - 1);
        if (!band_any(q0, q1, k0, k1, p.off, p.wl, p.wr)) return false;
    } else {
        if ((p.mode & kCausal) && j > rb) return false;
    }
    if ((p.mode & kSparse) && p.mask[static_cast<size_t>(rb) * p.nkb + j] == 0) return false;
    return true;
}

// Walks, in increasing order, the key blocks kept by at least one of the CTA's
// NQ query blocks (rb0, rb0 + 1).  Warp-collective: all 32 lanes call next().
template <int NQ, bool GENERAL>
struct KvIter {
    int base = -32;
    uint32_t b0 = 0, b1 = 0;
    __device__ __forceinline__ bool next(const FwdParams &p, int rb0, int &j, uint32_t &flags) {
        while ((b0 | b1) == 0u) {
            base += 32;
            if (base >= p.nkb) return false;
            const int jj = base + static_cast<int>(lane_id());
            b0 = __ballot_sync(0xffffffffu, block_kept<GENERAL>(p, rb0, jj));
            b1 = (NQ > 1) ? __ballot_sync(0xffffffffu, block_kept<GENERAL>(p, rb0 + 1, jj)) : 0u;
        }
        const uint32_t u = b0 | b1;
        const int b = __ffs(u) - 1;
        flags = ((b0 >> b) & 1u) | (((b1 >> b) & 1u) << 1);
        b0 &= ~(1u << b);
        b1 &= ~(1u << b);
        j = base + b;
        return true;
    }
};

template <int D, int NQ, int NSK, int NSV>
struct FwdCfg {
    static constexpr int kChunks = D / 64;              // 128-byte swizzle atoms along d
    static constexpr int kChunkBytes = 128 * 128;       // 128 rows x 128 bytes
    static constexpr int kTileBytes = 128 * D * 2;      // a 128-row tile of Q, K or V
    static constexpr int kQOff = 0;
    static constexpr int kKOff = kQOff + NQ * kTileBytes;
    static constexpr int kVOff = kKOff + NSK * kTileBytes;
    static constexpr int kBarOff = kVOff + NSV * kTileBytes;
    // barrier indices
    static constexpr int kBarQ = 0;
    static constexpr int kBarKFull = 1;
    static constexpr int kBarVFull = kBarKFull + NSK;
    static constexpr int kBarKEmpty = kBarVFull + NSV;
    static constexpr int kBarVEmpty = kBarKEmpty + NSK;
    static constexpr int kBarSFull = kBarVEmpty + NSV;
    static constexpr int kBarPFull = kBarSFull + NQ;
    static constexpr int kBarOFull = kBarPFull + NQ;
    static constexpr int kBarPFull2 = kBarOFull + NQ;   // P_t keys 64..127 in TMEM (kBarPFull: keys 0..63)
    static constexpr int kBarMmaDone = kBarPFull2 + NQ;
    // across work items (a CTA runs several in turn)
    static constexpr int kBarQEmpty = kBarMmaDone + 1;  // every S product of the item has read Q
    static constexpr int kBarOFree = kBarQEmpty + 1;    // [NQ] the epilogue has read O_t from TMEM
    static constexpr int kBarOStaged = kBarOFree + NQ;  // O of every tile staged in shared memory
    static constexpr int kBarStoreRead = kBarOStaged + 1;   // the TMA stores have read the staged O
    static constexpr int kNumBars = kBarStoreRead + 1;
    static constexpr int kMiscOff = kBarOff + kNumBars * 8;
    static constexpr int kSmemBytes = kMiscOff + 16 + 1024;   // + slack for 1 KB alignment
    static constexpr int kSoftmaxWarps = 4 * NQ;
    static constexpr int kWarpTma = kSoftmaxWarps;
    static constexpr int kWarpMma = kSoftmaxWarps + 1;
    // NQ = 2: V tiles come from their own producer warp, so that K tiles (more
    // stages, needed first) are never held up behind a V stage
    static constexpr int kWarpTmaV = NQ == 2 ? kSoftmaxWarps + 2 : kWarpTma;
    // NQ = 2: a third warpgroup (TMA, MMA, two idle warps) hands registers
    // to the softmax warpgroups (setmaxnreg: 2 x 128 x 216 + 128 x 72 =
    // 384 threads x 168 at launch).  NQ = 1: 6 warps, no reallocation.
    static constexpr int kThreads = NQ == 2 ? 384 : 32 * (kSoftmaxWarps + 2);
    static constexpr int kRegsSoftmax = 216;
    static constexpr int kRegsCtl = 72;
    static_assert(NQ == 1 || 2 * 128 * kRegsSoftmax + 128 * kRegsCtl <= 384 * 168, "register split");
    static constexpr int kOCol = 256;
    static_assert(D == 64 || D == 128 || D == 256, "head dim");
    static_assert(256 + NQ * D <= 512, "TMEM columns");
    static_assert(kSmemBytes <= 227 * 1024, "shared memory");
};

// Bounded wait that ignores the abort flag: used only to drain this CTA's own
// TMA loads / MMAs before it releases shared or tensor memory.
__device__ __forceinline__ void drain_bar(uint32_t bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return;
    const unsigned long long t0 = globaltimer();
    uint32_t it = 0;
    for (;;) {
        if (mbar_try_wait(bar, parity)) return;
        if ((++it & 31u) == 0 && globaltimer() - t0 > kTimeoutNs) {
            atomicCAS(&g_dev_status, 0, kErrTimeout);
            return;
        }
    }
}

// Work items: one per (batch-head, group of NQ query tiles), numbered query
// group major and batch-head minor, so that under causal masking the heaviest
// groups (the last query tiles) of every (b, h) come first.  A CTA runs the
// items r * G + c (r even) and r * G + G - 1 - c (r odd) of the grid of G
// CTAs, r = 0, 1, ...: heaviest first, and the back-and-forth order balances
// the sums of a decreasing sequence (at B=4 H=16 N=4096 causal, 1,024 items on
// 148 CTAs, the busiest CTA gets 1.02 x the mean work).
__device__ __forceinline__ int fwd_item(int r, int c, int G) {
    return r * G + ((r & 1) ? G - 1 - c : c);
}

template <int NQ>
__device__ __forceinline__ void fwd_decode(const FwdParams &p, int item, int &bh, int &rb0) {
    const int nqp = (p.nqb + NQ - 1) / NQ;
    bh = item % p.nbh;
    const int qi = item / p.nbh;
    rb0 = ((p.mode & kCausal) ? nqp - 1 - qi : qi) * NQ;
}

// The items a CTA runs, in turn r = 0, 1, ...  Dense problems: item
// fwd_item(r) of the grid above.  Packed variable-length batches (VARLEN):
// the same grid, sized by the longest sequence, walked in the same order with
// the positions past a sequence's own query groups skipped (v counts the
// positions walked); lp is then p with the item's sequence lengths, and the
// TMA coordinates of its rows are offset by qrow0 / krow0 in plane h.  Every
// role of the CTA walks the same items.
template <int NQ, bool VARLEN>
struct FwdWalk {
    int v = 0;
    int bh = 0, rb0 = 0;
    int qrow0 = 0, krow0 = 0, plane = 0;
    FwdParams lp;
    __device__ __forceinline__ const FwdParams &prm(const FwdParams &p) const {
        if constexpr (VARLEN) return lp;
        else return p;
    }
    __device__ __forceinline__ bool next(const FwdParams &p, int r, int cta, int G) {
        if constexpr (!VARLEN) {
            const int item = fwd_item(r, cta, G);
            if (item >= p.nitems) return false;
            fwd_decode<NQ>(p, item, bh, rb0);
            plane = bh;
            return true;
        } else {
            for (;;) {
                const int item = fwd_item(v++, cta, G);
                if (item >= p.nitems) return false;
                bh = item % p.nbh;
                const int qi = item / p.nbh;
                const int b = bh / p.H;
                plane = bh - b * p.H;
                const SeqSpan sq = seq_span(p.cu_q, b, p.total_q, p.Nq);
                const int nqb = (sq.len + 127) / 128;
                const int nqp = (nqb + NQ - 1) / NQ;
                if (qi >= nqp) continue;
                const SeqSpan sk = seq_span(p.cu_k, b, p.total_k, p.Nk);
                rb0 = ((p.mode & kCausal) ? nqp - 1 - qi : qi) * NQ;
                lp = p;
                lp.Nq = sq.len;
                lp.Nk = sk.len;
                lp.nqb = nqb;
                lp.nkb = (sk.len + 127) / 128;
                lp.off = sk.len - sq.len;
                qrow0 = sq.start;
                krow0 = sk.start;
                return true;
            }
        }
    }
};

// A CTA stays resident and runs its work items in turn.  Within an item the
// roles work as described at the top of this file; across items:
//   - the K producer loads the next item's Q once every S product of the
//     current item has completed (QEmpty), so the first S of the next item
//     follows the last P V of this one;
//   - O_t is staged in V ring stage t (every P V of the item has completed
//     when the epilogue runs) and written by TMA stores that the V producer
//     issues before it loads the next item's V tiles (OStaged, StoreRead);
//   - the MMA warp completes OFull_t of an item only after the epilogue of the
//     item before has read O_t from TMEM (OFree_t), so each of these barriers
//     completes once per item, in step with its waiter.
template <int D, int NQ, int NSK, int NSV, bool BF16, bool GENERAL, bool VARLEN = false>
__global__ void __launch_bounds__(FwdCfg<D, NQ, NSK, NSV>::kThreads, 1)
    fwd_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
               const __grid_constant__ CUtensorMap tmv, const __grid_constant__ CUtensorMap tmo, const FwdParams p) {
    using C = FwdCfg<D, NQ, NSK, NSV>;
    static_assert(NSV >= NQ, "O_t is staged in V stage t");
    static_assert(GENERAL || !VARLEN, "packed batches use the general band");
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = smem_u32(smem);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int cta = static_cast<int>(blockIdx.x);
    const int G = static_cast<int>(gridDim.x);

    auto bar = [&](int i) -> uint32_t { return sbase + C::kBarOff + 8u * i; };
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + C::kMiscOff);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::kMiscOff + 4);

    if (threadIdx.x == 0) {
        mbar_init(bar(C::kBarQ), 1);
        for (int s = 0; s < NSK; ++s) {
            mbar_init(bar(C::kBarKFull + s), 1);
            mbar_init(bar(C::kBarKEmpty + s), 1);
        }
        for (int s = 0; s < NSV; ++s) {
            mbar_init(bar(C::kBarVFull + s), 1);
            mbar_init(bar(C::kBarVEmpty + s), 1);
        }
        for (int t = 0; t < NQ; ++t) {
            mbar_init(bar(C::kBarSFull + t), 1);
            mbar_init(bar(C::kBarPFull + t), 128);
            mbar_init(bar(C::kBarPFull2 + t), 128);
            mbar_init(bar(C::kBarOFull + t), 1);
            mbar_init(bar(C::kBarOFree + t), 128);
        }
        mbar_init(bar(C::kBarMmaDone), 1);
        mbar_init(bar(C::kBarQEmpty), 1);
        mbar_init(bar(C::kBarOStaged), 32 * C::kSoftmaxWarps);
        mbar_init(bar(C::kBarStoreRead), 1);
        *abort_flag = 0;
        mbar_fence_init();
    }
    if (warp == C::kWarpMma) {
        tmem_alloc(smem_u32(tmem_holder), 512);
        tmem_relinquish();
    }
    if (warp == C::kWarpTma && lane == 0) {
        tma_prefetch_desc(&tmq);
        tma_prefetch_desc(&tmk);
        tma_prefetch_desc(&tmv);
        tma_prefetch_desc(&tmo);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    if (warp >= C::kSoftmaxWarps) {
        if constexpr (NQ == 2) setmaxnreg_dec<C::kRegsCtl>();
        if (warp == C::kWarpTma || warp == C::kWarpTmaV) {
            // ------------------------------------------------------------ producer(s)
            const bool do_k = warp == C::kWarpTma;
            const bool do_v = warp == C::kWarpTmaV;
            // TMA stores of item r's O tiles from V stages 0 .. NQ-1, once the
            // softmax warps have staged them; the stages are reloaded only
            // after the stores have read them
            auto store_item = [&](int r, int bh, int rb0, int nqb, int nq, int qrow0) -> bool {
                const bool ok = wait_bar(bar(C::kBarOStaged), r & 1, abort_flag);
                if (!ok) return ok;
                if constexpr (VARLEN) {
                    // a tile that ends inside the packed rows of the next
                    // sequence is written row by row with plain stores (a TMA
                    // store clips only at the end of the tensor)
                    for (int t = 0; t < NQ; ++t) {
                        const int rows = nq - (rb0 + t) * 128;
                        if (rb0 + t >= nqb || rows >= 128) continue;
                        const uint8_t *stage = smem + C::kVOff + t * C::kTileBytes;
                        uint8_t *dst = static_cast<uint8_t *>(p.o) +
                                       (static_cast<size_t>(qrow0 + (rb0 + t) * 128) * p.H + bh % p.H) * (D * 2);
                        for (int e = lane; e < rows * C::kChunks * 8; e += 32) {
                            const int rr = e / (C::kChunks * 8), c = (e >> 3) % C::kChunks, u = e & 7;
                            *reinterpret_cast<uint4 *>(dst + static_cast<size_t>(rr) * p.H * (D * 2) + c * 128 +
                                                       u * 16) =
                                *reinterpret_cast<const uint4 *>(stage + c * C::kChunkBytes + rr * 128 +
                                                                 ((u ^ (rr & 7)) << 4));
                        }
                    }
                    __syncwarp();
                }
                if (lane == 0) {
                    for (int t = 0; t < NQ; ++t) {
                        if (rb0 + t >= nqb) continue;
                        if (VARLEN && nq - (rb0 + t) * 128 < 128) continue;
                        for (int c = 0; c < C::kChunks; ++c)   // rows >= Nq are clipped
                            tma_store_3d(&tmo, sbase + C::kVOff + t * C::kTileBytes + c * C::kChunkBytes, c * 64,
                                         qrow0 + (rb0 + t) * 128, VARLEN ? bh % p.H : bh);
                    }
                    bulk_commit();
                    bulk_wait_read();
                    mbar_arrive(bar(C::kBarStoreRead));
                }
                __syncwarp();
                return ok;
            };
            int nk = 0, nv = 0;   // loads issued (all items)
            int nit = 0;          // items started
            int pbh = 0, prb0 = 0, pnqb = 0, pnq = 0, pq0 = 0;
            bool ok = true;
            FwdWalk<NQ, VARLEN> w;
            for (int r = 0; ok; ++r) {
                if (!w.next(p, r, cta, G)) break;
                const FwdParams &ip = w.prm(p);
                const int bh = w.bh, rb0 = w.rb0;
                if (do_v && r > 0) {
                    ok = store_item(r - 1, pbh, prb0, pnqb, pnq, pq0);
                    if (!ok) break;
                }
                if (do_k) {
                    if (r > 0) {
                        ok = wait_bar(bar(C::kBarQEmpty), (r - 1) & 1, abort_flag);
                        if (!ok) break;
                    }
                    if (lane == 0) {
                        int nq_valid = 0;
                        for (int t = 0; t < NQ; ++t) nq_valid += (rb0 + t < ip.nqb) ? 1 : 0;
                        mbar_arrive_expect_tx(bar(C::kBarQ), nq_valid * C::kTileBytes);
                        for (int t = 0; t < NQ; ++t) {
                            if (rb0 + t >= ip.nqb) continue;
                            for (int c = 0; c < C::kChunks; ++c)
                                tma_load_3d(sbase + C::kQOff + t * C::kTileBytes + c * C::kChunkBytes, &tmq,
                                            bar(C::kBarQ), c * 64, w.qrow0 + (rb0 + t) * 128, w.plane);
                        }
                    }
                    __syncwarp();
                }
                ++nit;
                KvIter<NQ, GENERAL> it;
                int j;
                uint32_t f;
                while (ok && it.next(ip, rb0, j, f)) {
                    if (do_k) {
                        const int s = nk % NSK;
                        ok = wait_bar(bar(C::kBarKEmpty + s), ((nk / NSK) & 1) ^ 1u, abort_flag);
                        if (!ok) break;
                        if (lane == 0) {
                            mbar_arrive_expect_tx(bar(C::kBarKFull + s), C::kTileBytes);
                            for (int c = 0; c < C::kChunks; ++c)
                                tma_load_3d(sbase + C::kKOff + s * C::kTileBytes + c * C::kChunkBytes, &tmk,
                                            bar(C::kBarKFull + s), c * 64, w.krow0 + j * 128, w.plane);
                        }
                        ++nk;
                    }
                    if (do_v) {
                        const int s = nv % NSV;
                        ok = wait_bar(bar(C::kBarVEmpty + s), ((nv / NSV) & 1) ^ 1u, abort_flag);
                        if (!ok) break;
                        if (lane == 0) {
                            mbar_arrive_expect_tx(bar(C::kBarVFull + s), C::kTileBytes);
                            for (int c = 0; c < C::kChunks; ++c)
                                tma_load_3d(sbase + C::kVOff + s * C::kTileBytes + c * C::kChunkBytes, &tmv,
                                            bar(C::kBarVFull + s), c * 64, w.krow0 + j * 128, w.plane);
                        }
                        ++nv;
                    }
                    __syncwarp();
                }
                pbh = bh;
                prb0 = rb0;
                pnqb = ip.nqb;
                pnq = ip.Nq;
                pq0 = w.qrow0;
            }
            // the last item's outputs
            if (do_v && ok && nit > 0) store_item(nit - 1, pbh, prb0, pnqb, pnq, pq0);
            // every issued load has landed before the CTA may exit
            if (do_k && nit > 0) drain_bar(bar(C::kBarQ), (nit - 1) & 1);
            for (int i = (nk > NSK ? nk - NSK : 0); i < nk; ++i)
                drain_bar(bar(C::kBarKFull + i % NSK), (i / NSK) & 1);
            for (int i = (nv > NSV ? nv - NSV : 0); i < nv; ++i)
                drain_bar(bar(C::kBarVFull + i % NSV), (i / NSV) & 1);
        } else if (warp == C::kWarpMma) {
            // ------------------------------------------------------------ MMA issuer
            const uint32_t leader = elect_one();   // the lane that issues tcgen05 ops
            constexpr uint32_t kIdescS = instr_desc_f16(128, 128, BF16, false, false);
            constexpr uint32_t kIdescO = instr_desc_f16(128, D, BF16, false, true);
            // descriptors built once; each instruction only offsets the start address
            const SmemDesc dQ = make_desc(sbase + C::kQOff, 16, 1024);
            const SmemDesc dK = make_desc(sbase + C::kKOff, 16, 1024);
            const SmemDesc dV = make_desc(sbase + C::kVOff, C::kChunkBytes, 1024);
            auto issue_s = [&](int t, int s) {
                const uint32_t d_tmem = tmem + 128u * t;
#pragma unroll
                for (int k = 0; k < D / 16; ++k) {
                    const uint32_t koff = (k >> 2) * C::kChunkBytes + (k & 3) * 32;
                    mma_ss(d_tmem, dQ.at(t * C::kTileBytes + koff), dK.at(s * C::kTileBytes + koff), kIdescS,
                           k > 0 ? 1u : 0u, leader);
                }
            };
            auto issue_pv = [&](int t, int s, bool acc, int k0, int k1) {
                const uint32_t d_tmem = tmem + C::kOCol + D * t;
                const uint32_t a_tmem = tmem + 128u * t;
#pragma unroll
                for (int k = k0; k < k1; ++k)
                    mma_ts(d_tmem, a_tmem + 8u * k, dV.at(s * C::kTileBytes + k * 2048), kIdescO,
                           (acc || k > 0) ? 1u : 0u, leader);
            };

            int kc = 0;        // K (= V) tiles consumed, all items
            int pc[NQ];        // P_t V products issued, all items (parity of PFull_t)
#pragma unroll
            for (int t = 0; t < NQ; ++t) pc[t] = 0;
            bool ok = true;
            FwdWalk<NQ, VARLEN> w;
            for (int r = 0; ok; ++r) {
                if (!w.next(p, r, cta, G)) break;
                const FwdParams &ip = w.prm(p);
                const int rb0 = w.rb0;
                int ci[NQ];    // P_t V products of this item (accumulate after the first)
#pragma unroll
                for (int t = 0; t < NQ; ++t) ci[t] = 0;
                KvIter<NQ, GENERAL> it;
                int j, jn;
                uint32_t f, fn;
                bool have = it.next(ip, rb0, j, f);
                ok = wait_bar(bar(C::kBarQ), r & 1, abort_flag);
                if (!ok) break;
                tc_fence_after();
                if (have) {
                    const int s0 = kc % NSK;
                    ok = wait_bar(bar(C::kBarKFull + s0), (kc / NSK) & 1, abort_flag);
                    if (!ok) break;
                    tc_fence_after();
                    for (int t = 0; t < NQ; ++t)
                        if ((f >> t) & 1u) {
                            issue_s(t, s0);
                            mma_commit(bar(C::kBarSFull + t), leader);
                        }
                    mma_commit(bar(C::kBarKEmpty + s0), leader);
                    __syncwarp();
                } else {
                    mma_commit(bar(C::kBarQEmpty), leader);   // no S product reads this Q
                    __syncwarp();
                }
                int u = 0;
                while (ok && have) {
                    const int vi = kc + u;                 // V tile of this key tile
                    const int s = vi % NSV;
                    const uint32_t ph = (vi / NSV) & 1;
                    const int ki = kc + u + 1;             // K tile of the next key tile
                    const int sn = ki % NSK;
                    const uint32_t phn = (ki / NSK) & 1;
                    const bool have_n = it.next(ip, rb0, jn, fn);
                    if (!have_n) {
                        // every S product of the item is issued: Q may be replaced
                        mma_commit(bar(C::kBarQEmpty), leader);
                        __syncwarp();
                    }
                    ok = wait_bar(bar(C::kBarVFull + s), ph, abort_flag);
                    if (!ok) break;
                    tc_fence_after();
                    bool k_ready = false;
#pragma unroll
                    for (int t = 0; t < NQ; ++t) {
                        if ((f >> t) & 1u) {
                            ok = wait_bar(bar(C::kBarPFull + t), pc[t] & 1, abort_flag);
                            if (!ok) break;
                            tc_fence_after();
                            issue_pv(t, s, ci[t] > 0, 0, 4);
                            __syncwarp();
                            ok = wait_bar(bar(C::kBarPFull2 + t), pc[t] & 1, abort_flag);
                            if (!ok) break;
                            tc_fence_after();
                            issue_pv(t, s, ci[t] > 0, 4, 8);
                            __syncwarp();
                            ++pc[t];
                            ++ci[t];
                        }
                        // V_j is read by no later product: its stage is released when
                        // the last P V completes, not after S of the next key tile too
                        // (measured: +5.6 % at d = 256, where V has one stage; +0.3 to
                        // +1.4 % at d = 128)
                        if (t == NQ - 1) mma_commit(bar(C::kBarVEmpty + s), leader);
                        if (have_n && ((fn >> t) & 1u)) {
                            if (!k_ready) {
                                ok = wait_bar(bar(C::kBarKFull + sn), phn, abort_flag);
                                if (!ok) break;
                                tc_fence_after();
                                k_ready = true;
                            }
                            issue_s(t, sn);
                            mma_commit(bar(C::kBarSFull + t), leader);
                            __syncwarp();
                        }
                    }
                    if (!ok) break;
                    if (have_n) mma_commit(bar(C::kBarKEmpty + sn), leader);
                    __syncwarp();
                    j = jn;
                    f = fn;
                    have = have_n;
                    ++u;
                }
                if (!ok) break;
                kc += u;
                // O_t of this item is final once the products above complete;
                // the item before must have read O_t first (one completion of
                // OFull_t per item, in step with the epilogue that waits on it)
                for (int t = 0; t < NQ; ++t) {
                    if (r > 0) {
                        ok = wait_bar(bar(C::kBarOFree + t), (r - 1) & 1, abort_flag);
                        if (!ok) break;
                    }
                    mma_commit(bar(C::kBarOFull + t), leader);
                    __syncwarp();
                }
            }
            mma_commit(bar(C::kBarMmaDone), leader);
            __syncwarp();
            drain_bar(bar(C::kBarMmaDone), 0);
        }
    } else {
        if constexpr (NQ == 2) setmaxnreg_inc<C::kRegsSoftmax>();
        // ------------------------------------------------------------ softmax
        const int t = warp >> 2;
        const int wq = warp & 3;
        const int row_local = wq * 32 + lane;
        const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
        const uint32_t tS = tmem + lane_off + 128u * t;
        const uint32_t tO = tmem + lane_off + C::kOCol + D * t;
        const float c = p.scale_log2;
        int sc = 0;            // S_t products consumed, all items (parity of SFull_t)
        bool ok = true;
        FwdWalk<NQ, VARLEN> w;
        for (int ri = 0; ok; ++ri) {
            if (!w.next(p, ri, cta, G)) break;
            const FwdParams &ip = w.prm(p);
            const int bh = w.bh, rb0 = w.rb0;
            const int rb = rb0 + t;
            const int row = rb * 128 + row_local;
            float m = -INFINITY, l = 0.f, l_r = 0.f;
            int cnt = 0;
            // does this row see any key?  Taken from the band limits of the tiles
            // it meets, not from m or l: a row that sees no key keeps m = -inf
            // only while every masked score stays -inf, and the polynomial exp2
            // gives masked scores 2^-125 instead of 0
            bool seen = false;
            KvIter<NQ, GENERAL> it;
            int j;
            uint32_t f;
            while (it.next(ip, rb0, j, f)) {
                if (!((f >> t) & 1u)) continue;
                ok = wait_bar(bar(C::kBarSFull + t), sc & 1, abort_flag);
                if (!ok) break;
                ++sc;
                tc_fence_after();
                uint32_t r[128];
#pragma unroll
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    tmem_ld32(tS + 32 * q, *reinterpret_cast<uint32_t(*)[32]>(&r[32 * q]));
                tmem_wait_ld(r);
                // the scores as floats: a copy, not a float* view of r (reading
                // the asm-written integers through another type is undefined and
                // let stale register values into the row max)
                float sv[128];
#pragma unroll
                for (int k = 0; k < 128; ++k) sv[k] = __uint_as_float(r[k]);
                // this row's visible keys within the tile: [lo, hi]
                int lo, hi, rk = 0;
                if constexpr (GENERAL) {
                    rk = row + ip.off - j * 128;     // |values| < 2^30 (Nq, Nk <= 2^28)
                    lo = max(rk - p.wl, -1);
                    hi = min(min(rk + p.wr, ip.Nk - 1 - j * 128), 128);
                } else {
                    lo = -1;
                    hi = 127;
                    if ((p.mode & kCausal) && j == rb) hi = row_local;                    // diagonal tile
                    if (j == p.nkb - 1 && (p.Nk & 127)) hi = min(hi, (p.Nk & 127) - 1);  // key tail
                }
                seen |= max(lo, 0) <= min(hi, 127);
                if (GENERAL && p.alibi) {
                    // score + bias / scale, bias = -slope |row + off - key|
                    const float sl = -p.alibi[bh % p.H] / p.scale;
                    const float base = static_cast<float>(rk);
#pragma unroll
                    for (int k = 0; k < 128; ++k) sv[k] = fmaf(sl, fabsf(base - static_cast<float>(k)), sv[k]);
                }
                if (__any_sync(0xffffffffu, lo > 0 || hi < 127)) {
#pragma unroll
                    for (int k = 0; k < 128; ++k)
                        if (k < lo || k > hi) sv[k] = -INFINITY;
                }
                // row max: four independent chains, two scores per step (fmax3)
                float mx0 = sv[0], mx1 = sv[1], mx2 = sv[2], mx3 = sv[3];
#pragma unroll
                for (int k = 4; k < 128; k += 8) {
                    mx0 = fmax3(mx0, sv[k], sv[k + 1]);
                    mx1 = fmax3(mx1, sv[k + 2], sv[k + 3]);
                    mx2 = fmax3(mx2, sv[k + 4], sv[k + 5]);
                    mx3 = fmax3(mx3, sv[k + 6], sv[k + 7]);
                }
                const float mx = fmax3(mx0, mx1, fmaxf(mx2, mx3));
                const float m_cand = fmaxf(m, mx * c);
                const bool grow = m_cand > m + 8.0f;    // lazy: keep m unless it moves by > 2^8
                const float m_new = grow ? m_cand : m;
                const float alpha = grow ? ex2(m - m_new) : 1.0f;
                const float m_use = (m_new == -INFINITY) ? 0.0f : m_new;
                if (cnt > 0 && __any_sync(0xffffffffu, grow)) {
                    // S_t's completion implies the previous O_t += P V finished
#pragma unroll 1
                    for (int q = 0; q < D / 32; ++q) {
                        uint32_t o[32];
                        tmem_ld32_wait(tO + 32 * q, o);
#pragma unroll
                        for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
                        tmem_st32(tO + 32 * q, o);
                    }
                }
                // P = 2^(s c - m).  kPolyPairs of every 8 pairs may go to the FMA
                // pipe (polynomial) instead of the special-function unit.  Measured
                // on B200 with the persistent kernel: slower at every share tried
                // (d = 128: one of eight pairs -4 %, two -7 %; d = 64: two of
                // eight -2 %), so every pair uses the special-function unit.  (An
                // earlier parity failure of the polynomial build was the
                // three-input max of the row-max tree, now two-input, and rows
                // with no visible key are recognised by their band limits.)
                constexpr int kPolyPairs = 0;
                float2 acc[4], acc_r[4];
#pragma unroll
                for (int a4 = 0; a4 < 4; ++a4) acc[a4] = acc_r[a4] = make_float2(0.f, 0.f);
                const float2 cc = make_float2(c, c), mm = make_float2(-m_use, -m_use);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    uint32_t pk[16];
#pragma unroll
                    for (int k = 0; k < 16; ++k) {
                        const int g = 16 * q + k;
                        const float2 x = ffma2(make_float2(sv[2 * g], sv[2 * g + 1]), cc, mm);
                        float2 pr;
                        if ((g & 7) >= 8 - kPolyPairs) {
                            pr = exp2_poly2(x);
                        } else {
                            pr.x = ex2(x.x);
                            pr.y = ex2(x.y);
                        }
                        pk[k] = pack2<BF16>(pr.x, pr.y);
                        acc[k & 3] = fadd2(acc[k & 3], pr);
                        if constexpr (BF16) {
                            // O is normalised by the sum of the same rounded P the
                            // tensor core multiplies (a row dominated by one key then
                            // comes out exact); LSE keeps the unrounded sum
                            acc_r[k & 3] = fadd2(acc_r[k & 3], unpack2<true>(pk[k]));
                        }
                    }
                    tmem_st16(tS + 16 * q, pk);
                    if (q == 1) {
                        // the first 64 keys of P_t are in TMEM: the MMA warp can start
                        // O_t += P_t V on them while the second half is computed
                        tmem_st_wait();
                        tc_fence_before();
                        mbar_arrive(bar(C::kBarPFull + t));
                    }
                }
                const float2 s01 = fadd2(fadd2(acc[0], acc[1]), fadd2(acc[2], acc[3]));
                const float sum = s01.x + s01.y;
                float sum_r = 0.f;
                if constexpr (BF16) {
                    const float2 r01 = fadd2(fadd2(acc_r[0], acc_r[1]), fadd2(acc_r[2], acc_r[3]));
                    sum_r = r01.x + r01.y;
                }
                l = l * alpha + sum;
                if constexpr (BF16) l_r = l_r * alpha + sum_r;
                m = m_new;
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(bar(C::kBarPFull2 + t));
                ++cnt;
            }
            if (!ok) break;
            // ---------------------------------------------------------- epilogue
            ok = wait_bar(bar(C::kBarOFull + t), ri & 1, abort_flag);
            if (!ok) break;
            tc_fence_after();
            // O_t is staged in V stage t (every P V of the item has completed)
            // once the previous item's stores have read it, as 128-byte-swizzled
            // 64-column chunks for the V producer's TMA stores
            if (ri > 0) {
                ok = wait_bar(bar(C::kBarStoreRead), (ri - 1) & 1, abort_flag);
                if (!ok) break;
            }
            if (rb < ip.nqb) {
                uint8_t *stage = smem + C::kVOff + t * C::kTileBytes;
                const float l_o = BF16 ? l_r : l;
                // a row that saw no key: O = 0, LSE = -inf
                const float inv_l = (seen && l_o > 0.f) ? 1.0f / l_o : 0.0f;
#pragma unroll 1
                for (int q = 0; q < D / 32; ++q) {
                    uint32_t o[32];
                    if (cnt > 0) {
                        tmem_ld32_wait(tO + 32 * q, o);
                    } else {
#pragma unroll
                        for (int k = 0; k < 32; ++k) o[k] = 0u;
                    }
                    uint32_t pk[16];
#pragma unroll
                    for (int k = 0; k < 16; ++k)
                        pk[k] = pack2<BF16>(__uint_as_float(o[2 * k]) * inv_l,
                                            __uint_as_float(o[2 * k + 1]) * inv_l);
                    uint8_t *srow = stage + (q >> 1) * C::kChunkBytes + row_local * 128;
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const int u = (q & 1) * 4 + k;   // 16-byte unit within the 128-byte row
                        *reinterpret_cast<uint4 *>(srow + ((u ^ (row_local & 7)) << 4)) =
                            make_uint4(pk[4 * k], pk[4 * k + 1], pk[4 * k + 2], pk[4 * k + 3]);
                    }
                }
                if (row < ip.Nq) {
                    const float lse = (seen && l > 0.f) ? (m + log2f(l)) * 0.69314718055994531f : -INFINITY;
                    if constexpr (VARLEN)
                        p.lse[static_cast<size_t>(w.plane) * p.total_q + w.qrow0 + row] = lse;
                    else
                        p.lse[static_cast<size_t>(bh) * p.Nq + row] = lse;
                }
            }
            tc_fence_before();
            mbar_arrive(bar(C::kBarOFree + t));     // O_t read: the next item may complete OFull_t
            fence_async_smem();
            mbar_arrive(bar(C::kBarOStaged));      // staged O visible to the TMA stores
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
