// fa_fwd_fp8.cuh -- FP8 forward with block quantisation and incoherent
// processing, sm_100a.
//
// "FlashAttention 深度解析" section 四: FlashAttention-3 adds FP8 block
// quantisation, with incoherent processing to lower the FP8 error.  The
// definitions (the readings of that sentence) are:
//   rotation    Q and K are multiplied by M = diag(signs) H_d / sqrt(d) (H_d
//               the Sylvester Hadamard matrix, signs +-1); Q M (K M)^T = Q K^T,
//               and an outlier channel is spread over all d channels.
//   quantiser   E4M3 codes with one scale amax / 448 per 128-row block of Q
//               and of K, and one per head for V; code = E4M3(x * (448 / amax))
//               rounded to nearest even, saturating at 448.  The rotation and
//               the quantiser run in fp32 one IEEE operation at a time in a
//               fixed order (butterfly stages h = 1, 2, ..., d/2 on pairs
//               (c, c + h) -> (a + b, a - b), then one multiply by 1/sqrt(d)),
//               so the codes are fully determined by the inputs.
//   attention   S = scale * sq_i * sk_j * Q8 K8^T (tcgen05 kind::f8f6f4, fp32
//               accumulation), online softmax in fp32 as in the 16-bit
//               forward, P rounded to E4M3 and O += P8 V8 (FP8 again), O
//               divided by the sum of the rounded P and multiplied by sv.
//
// Kernels:
//   fp8_quant_kernel   pass 0: one CTA per (128-row block, (b, h), tensor):
//                      Q and K are rotated (when signs are given) and
//                      quantised with the block's scale; V blocks only report
//                      their amax.  pass 1: V blocks are quantised with the
//                      head's amax.  One warp per row: each lane holds d/32
//                      consecutive channels; butterflies below d/32 run in the
//                      lane, the others across lanes with shuffles.
//   fp8_vscale_kernel  the head's V scale, written to every block slot.
//   fwd8_kernel        the forward of fa_fwd.cuh (dense or causal) on E4M3
//                      operands: d = 64 and 128 with two 128-row query tiles
//                      per CTA, d = 256 with one (its O accumulator takes 256
//                      TMEM columns).  Q8, K8, V8 tiles are swizzle atoms of
//                      128-byte rows (two per tile at d = 256; 64-byte rows
//                      with the 64-byte swizzle at d = 64), P8 takes 32 TMEM
//                      columns (four codes per column) over S, O tiles are
//                      staged in the finished K ring and written by TMA stores.
#pragma once

#include "fa_fwd.cuh"

namespace fa {

// ---------------------------------------------------------------------------
// quantiser
// ---------------------------------------------------------------------------
struct QuantParams {
    const void *src[3];   // Q, K, V: [BH][N][D] 16-bit
    uint8_t *dst[3];      // E4M3 codes [BH][N][D]
    float *scales[3];     // [BH][nb]; V: block amax after pass 0, the head's scale after fp8_vscale_kernel
    const float *signs;   // [D] of +-1 (rotation of Q and K) or null
    float rnorm;          // (float)(1 / sqrt(D))
    int N, nb;
};

template <int D>
struct QuantCfg {
    static constexpr int kWarps = D == 256 ? 16 : 8;
    static constexpr int kThreads = 32 * kWarps;
    static constexpr int kRows = 128 / kWarps;   // rows per warp
    static constexpr int E = D / 32;             // channels per lane
};

template <int D, bool BF16>
__global__ void __launch_bounds__(QuantCfg<D>::kThreads)
    fp8_quant_kernel(const QuantParams p, int pass) {
    using C = QuantCfg<D>;
    constexpr int E = C::E;
    __shared__ float red[C::kWarps];
    // one-dimensional grid over ((b, h), block); blockIdx.y selects Q, K, V in pass 0
    const int z = pass == 0 ? static_cast<int>(blockIdx.y) : 2;
    const int b = static_cast<int>(blockIdx.x % static_cast<unsigned>(p.nb));
    const long long bh = blockIdx.x / static_cast<unsigned>(p.nb);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const bool rotate = z < 2 && p.signs != nullptr;
    // operands picked with selects (indexing the parameter arrays would copy them to local memory)
    const uint16_t *src = static_cast<const uint16_t *>(z == 0 ? p.src[0] : (z == 1 ? p.src[1] : p.src[2]));
    // every row's load is issued before any arithmetic (HBM-bound: bytes in flight)
    uint32_t raw[C::kRows][E / 2];
#pragma unroll
    for (int r = 0; r < C::kRows; ++r) {
        const int row = b * 128 + warp * C::kRows + r;
        const uint16_t *s = src + (static_cast<size_t>(bh) * p.N + row) * D + lane * E;
        if (row < p.N) {
            if constexpr (E == 2) {
                raw[r][0] = *reinterpret_cast<const uint32_t *>(s);
            } else if constexpr (E == 4) {
                const uint2 w = *reinterpret_cast<const uint2 *>(s);
                raw[r][0] = w.x;
                raw[r][1] = w.y;
            } else {
                const uint4 w = *reinterpret_cast<const uint4 *>(s);
                raw[r][0] = w.x;
                raw[r][1] = w.y;
                raw[r][2] = w.z;
                raw[r][3] = w.w;
            }
        } else {
#pragma unroll
            for (int e = 0; e < E / 2; ++e) raw[r][e] = 0u;   // outside the tensor: not part of the block
        }
    }
    float x[C::kRows][E];
    float sg[E];
#pragma unroll
    for (int e = 0; e < E; ++e) sg[e] = rotate ? p.signs[lane * E + e] : 1.0f;
    float amax = 0.0f;
#pragma unroll
    for (int r = 0; r < C::kRows; ++r) {
#pragma unroll
        for (int e = 0; e < E; e += 2) {
            const float2 v = unpack2<BF16>(raw[r][e / 2]);
            x[r][e] = v.x;
            x[r][e + 1] = v.y;
        }
        if (rotate) {
#pragma unroll
            for (int e = 0; e < E; ++e) x[r][e] = x[r][e] * sg[e];
#pragma unroll
            for (int h = 1; h < E; h <<= 1)                // butterflies inside the lane
#pragma unroll
                for (int e = 0; e < E; ++e)
                    if (!(e & h)) {
                        const float a = x[r][e], c = x[r][e + h];
                        x[r][e] = a + c;
                        x[r][e + h] = a - c;
                    }
#pragma unroll
            for (int h = E; h < D; h <<= 1) {              // across lanes: lane ^ (h / E)
                // lower lane: x + y; upper lane: y - x, as one exactly rounded
                // fma(+-1, x, y) (the same result as the add or the subtraction)
                const float sgn = (lane & (h / E)) == 0 ? 1.0f : -1.0f;
#pragma unroll
                for (int e = 0; e < E; ++e) {
                    const float y = __shfl_xor_sync(0xffffffffu, x[r][e], h / E);
                    x[r][e] = fmaf(sgn, x[r][e], y);
                }
            }
#pragma unroll
            for (int e = 0; e < E; ++e) x[r][e] = x[r][e] * p.rnorm;
        }
#pragma unroll
        for (int e = 0; e < E; ++e) amax = fmaxf(amax, fabsf(x[r][e]));
    }
    float *sc = (z == 0 ? p.scales[0] : (z == 1 ? p.scales[1] : p.scales[2])) + bh * p.nb;
    if (pass == 0) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        if (lane == 0) red[warp] = amax;
        __syncthreads();
        amax = red[0];
#pragma unroll
        for (int w = 1; w < C::kWarps; ++w) amax = fmaxf(amax, red[w]);
        if (z == 2) {                                      // V: report the block amax only
            if (threadIdx.x == 0) sc[b] = amax;
            return;
        }
        if (threadIdx.x == 0) sc[b] = amax > 0.0f ? amax / 448.0f : 1.0f;
    } else {
        if (warp == 0) {                                   // V: the head's amax (max of the block amaxes)
            float hm = 0.0f;
            for (int k = lane; k < p.nb; k += 32) hm = fmaxf(hm, sc[k]);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) hm = fmaxf(hm, __shfl_xor_sync(0xffffffffu, hm, o));
            if (lane == 0) red[0] = hm;
        }
        __syncthreads();
        amax = red[0];
    }
    const float inv = amax > 0.0f ? 448.0f / amax : 1.0f;
    uint8_t *dst = z == 0 ? p.dst[0] : (z == 1 ? p.dst[1] : p.dst[2]);
#pragma unroll
    for (int r = 0; r < C::kRows; ++r) {
        const int row = b * 128 + warp * C::kRows + r;
        if (row >= p.N) continue;
        uint32_t pr[(E + 1) / 2];
#pragma unroll
        for (int e = 0; e < E; e += 2) pr[e / 2] = e4m3x2(x[r][e] * inv, x[r][e + 1] * inv);
        uint8_t *d8 = dst + (static_cast<size_t>(bh) * p.N + row) * D + lane * E;
        if constexpr (E == 2) {
            *reinterpret_cast<uint16_t *>(d8) = static_cast<uint16_t>(pr[0]);
        } else if constexpr (E == 4) {
            *reinterpret_cast<uint32_t *>(d8) = pr[0] | (pr[1] << 16);
        } else {
            *reinterpret_cast<uint2 *>(d8) = make_uint2(pr[0] | (pr[1] << 16), pr[2] | (pr[3] << 16));
        }
    }
}

// The head's V scale amax / 448 (amax = the largest block amax), written to
// every block slot of the head; one thread per (b, h).
__global__ void fp8_vscale_kernel(float *sv, int nb, long long BH) {
    const long long bh = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (bh >= BH) return;
    float *s = sv + bh * nb;
    float amax = 0.0f;
    for (int k = 0; k < nb; ++k) amax = fmaxf(amax, s[k]);
    const float scale = amax > 0.0f ? amax / 448.0f : 1.0f;
    for (int k = 0; k < nb; ++k) s[k] = scale;
}

// ---------------------------------------------------------------------------
// FP8 forward (d = 64, 128, 256)
// ---------------------------------------------------------------------------
struct Fwd8Params {
    float *lse;               // [BH][N]
    const float *sq, *sk;     // [BH][nb] block scales of Q8 and K8
    const float *sv;          // [BH][nb] the head's V scale (every slot)
    int N, nb, nbh;
    int causal;
    float scale_log2;         // scale * log2(e)
};

template <int D>
struct Fwd8Cfg {
    // d = 64, 128: two 128-row query tiles per CTA; d = 256: one (the O
    // accumulator takes 256 TMEM columns)
    static constexpr int NQ = D <= 128 ? 2 : 1;
    static constexpr int NSK = D == 256 ? 3 : 6, NSV = D == 256 ? 2 : 4;
    // rows of E4M3 codes in swizzle atoms of 128 bytes (d = 64: 64 bytes, the
    // 64-byte swizzle); a 128-row tile is D / kRowBytes atoms kAtom apart
    static constexpr int kRowBytes = D < 128 ? D : 128;
    static constexpr int kAtom = 128 * kRowBytes;
    static constexpr int kTileBytes = 128 * D;
    static constexpr int kOChunk = 128 * 128;           // 64 16-bit columns of a 128-row O tile
    static constexpr int kQOff = 0;
    static constexpr int kKOff = kQOff + NQ * kTileBytes;
    static constexpr int kVOff = kKOff + NSK * kTileBytes;
    static constexpr int kBarOff = kVOff + NSV * kTileBytes;
    static constexpr int kBarQ = 0;
    static constexpr int kBarKFull = 1;
    static constexpr int kBarVFull = kBarKFull + NSK;
    static constexpr int kBarKEmpty = kBarVFull + NSV;
    static constexpr int kBarVEmpty = kBarKEmpty + NSK;
    static constexpr int kBarSFull = kBarVEmpty + NSV;
    static constexpr int kBarPFull = kBarSFull + NQ;
    static constexpr int kBarOFull = kBarPFull + NQ;
    static constexpr int kBarMmaDone = kBarOFull + NQ;
    static constexpr int kNumBars = kBarMmaDone + 1;
    static constexpr int kMiscOff = kBarOff + kNumBars * 8;
    static constexpr int kSmemBytes = kMiscOff + 16 + 1024;
    static constexpr int kSoftmaxWarps = 4 * NQ;
    // softmax warpgroups, then one of TMA (K), MMA, TMA (V) and an idle warp
    static constexpr int kThreads = 32 * (kSoftmaxWarps + 4);
    static constexpr int kWarpTma = kSoftmaxWarps, kWarpMma = kSoftmaxWarps + 1, kWarpTmaV = kSoftmaxWarps + 2;
    static constexpr int kRegsSoftmax = 216, kRegsCtl = 72;   // NQ = 2 only (setmaxnreg)
    static constexpr int kOCol = 128 * NQ;
    static_assert(NQ == 1 || 2 * 128 * kRegsSoftmax + 128 * kRegsCtl <= 384 * 168, "register split");
    static_assert(NQ * (D / 64) * kOChunk <= NSK * kTileBytes, "O staging fits the K ring");
    static_assert(kOCol + NQ * D <= 512, "TMEM columns");
    static_assert(D == 64 || D == 128 || D == 256, "head dim");
    static_assert(kSmemBytes <= 227 * 1024, "shared memory");
};

// Key blocks of a causal or dense square problem seen by query block pair (rb0, rb0 + 1):
// j < min(nb, rb0 + 2) (causal) or j < nb; flags bit t: block j is seen by tile t.
template <int NQ>
__device__ __forceinline__ uint32_t fwd8_flags(const Fwd8Params &p, int rb0, int j) {
    uint32_t f = 0;
#pragma unroll
    for (int t = 0; t < NQ; ++t)
        if (rb0 + t < p.nb && (!p.causal || j <= rb0 + t)) f |= 1u << t;
    return f;
}

template <int D, bool BF16>
__global__ void __launch_bounds__(Fwd8Cfg<D>::kThreads, 1)
    fwd8_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                const __grid_constant__ CUtensorMap tmv, const __grid_constant__ CUtensorMap tmo,
                const Fwd8Params p) {
    using C = Fwd8Cfg<D>;
    constexpr int NQ = C::NQ, NSK = C::NSK, NSV = C::NSV;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = smem_u32(smem);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    // one-dimensional grid, (batch, head) minor, heaviest query pairs first under causal
    const int nqp = (p.nb + NQ - 1) / NQ;
    const int bh = static_cast<int>(blockIdx.x % static_cast<unsigned>(p.nbh));
    const int qi = static_cast<int>(blockIdx.x / static_cast<unsigned>(p.nbh));
    const int rb0 = (p.causal ? nqp - 1 - qi : qi) * NQ;
    const int nkb = p.causal ? min(p.nb, rb0 + NQ) : p.nb;   // key blocks this CTA visits: 0 .. nkb-1

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
            mbar_init(bar(C::kBarOFull + t), 1);
        }
        mbar_init(bar(C::kBarMmaDone), 1);
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
            // ------------------------------------------------------------ producers
            const bool do_k = warp == C::kWarpTma;
            if (do_k && lane == 0) {
                int nq_valid = 0;
                for (int t = 0; t < NQ; ++t) nq_valid += (rb0 + t < p.nb) ? 1 : 0;
                mbar_arrive_expect_tx(bar(C::kBarQ), nq_valid * C::kTileBytes);
                for (int t = 0; t < NQ; ++t)
                    if (rb0 + t < p.nb)
                        for (int a = 0; a < D / C::kRowBytes; ++a)
                            tma_load_3d(sbase + C::kQOff + t * C::kTileBytes + a * C::kAtom, &tmq, bar(C::kBarQ),
                                        a * C::kRowBytes, (rb0 + t) * 128, bh);
            }
            __syncwarp();
            const int NS = do_k ? NSK : NSV;
            const int full0 = do_k ? C::kBarKFull : C::kBarVFull;
            const int empty0 = do_k ? C::kBarKEmpty : C::kBarVEmpty;
            const uint32_t off0 = do_k ? C::kKOff : C::kVOff;
            const CUtensorMap *map = do_k ? &tmk : &tmv;
            int n = 0;
            for (int j = 0; j < nkb; ++j, ++n) {
                const int s = n % NS;
                if (!wait_bar(bar(empty0 + s), ((n / NS) & 1) ^ 1u, abort_flag)) break;
                if (lane == 0) {
                    mbar_arrive_expect_tx(bar(full0 + s), C::kTileBytes);
                    for (int a = 0; a < D / C::kRowBytes; ++a)
                        tma_load_3d(sbase + off0 + s * C::kTileBytes + a * C::kAtom, map, bar(full0 + s),
                                    a * C::kRowBytes, j * 128, bh);
                }
                __syncwarp();
            }
            if (do_k) drain_bar(bar(C::kBarQ), 0);
            for (int x = (n > NS ? n - NS : 0); x < n; ++x) drain_bar(bar(full0 + x % NS), (x / NS) & 1);
        } else if (warp == C::kWarpMma) {
            // ------------------------------------------------------------ MMA issuer
            const uint32_t leader = elect_one();
            constexpr uint32_t kIdS = instr_desc_e4m3(128, 128, false, false);
            constexpr uint32_t kIdO = instr_desc_e4m3(128, D, false, true);
            // 8-row groups of the swizzle atoms are 8 rows apart (sbo); V8 is the
            // MN-major B operand of P V, its atoms along d kAtom apart (lbo)
            constexpr uint32_t kSbo = 8 * C::kRowBytes;
            auto desc = [&](uint32_t a, uint32_t lbo) { return D == 64 ? make_desc_sw64(a, lbo, kSbo) : make_desc(a, lbo, kSbo); };
            const SmemDesc dQ = desc(sbase + C::kQOff, 16);
            const SmemDesc dK = desc(sbase + C::kKOff, 16);
            const SmemDesc dV = desc(sbase + C::kVOff, C::kAtom);
            auto issue_s = [&](int t, int s) {   // S_t = Q8_t K8_j^T: K = 32 steps along the rows of each atom
#pragma unroll
                for (int k = 0; k < D / 32; ++k) {
                    constexpr int kSteps = C::kRowBytes / 32;   // K steps per atom
                    const uint32_t o = (k / kSteps) * C::kAtom + 32 * (k % kSteps);
                    mma8_ss(tmem + 128u * t, dQ.at(t * C::kTileBytes + o), dK.at(s * C::kTileBytes + o), kIdS,
                            k > 0 ? 1u : 0u, leader);
                }
            };
            auto issue_pv = [&](int t, int s, bool acc) {   // O_t += P8_t V8_j: keys 32k.. in P8 columns 8k..
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    mma8_ts(tmem + C::kOCol + D * t, tmem + 128u * t + 8u * k,
                            dV.at(s * C::kTileBytes + k * 32 * C::kRowBytes), kIdO, (acc || k > 0) ? 1u : 0u, leader);
            };
            int cnt[NQ];
#pragma unroll
            for (int t = 0; t < NQ; ++t) cnt[t] = 0;
            bool ok = true;
            if (nkb > 0) {
                ok = wait_bar(bar(C::kBarQ), 0, abort_flag) && wait_bar(bar(C::kBarKFull), 0, abort_flag);
                if (ok) {
                    tc_fence_after();
                    const uint32_t f = fwd8_flags<NQ>(p, rb0, 0);
                    for (int t = 0; t < NQ; ++t)
                        if ((f >> t) & 1u) {
                            issue_s(t, 0);
                            mma_commit(bar(C::kBarSFull + t), leader);
                        }
                    mma_commit(bar(C::kBarKEmpty), leader);
                    __syncwarp();
                }
            }
            for (int u = 0; ok && u < nkb; ++u) {
                const int s = u % NSV;
                const bool have_n = u + 1 < nkb;
                const uint32_t f = fwd8_flags<NQ>(p, rb0, u);
                const uint32_t fn = have_n ? fwd8_flags<NQ>(p, rb0, u + 1) : 0u;
                const int sn = (u + 1) % NSK;
                ok = wait_bar(bar(C::kBarVFull + s), (u / NSV) & 1, abort_flag);
                if (!ok) break;
                tc_fence_after();
                bool k_ready = false;
                for (int t = 0; t < NQ; ++t) {
                    if ((f >> t) & 1u) {
                        ok = wait_bar(bar(C::kBarPFull + t), cnt[t] & 1, abort_flag);
                        if (!ok) break;
                        tc_fence_after();
                        issue_pv(t, s, cnt[t] > 0);
                        __syncwarp();
                        ++cnt[t];
                    }
                    // V_j's stage is released when the last P V completes (as in the
                    // 16-bit forward)
                    if (t == NQ - 1) mma_commit(bar(C::kBarVEmpty + s), leader);
                    if ((fn >> t) & 1u) {
                        if (!k_ready) {
                            ok = wait_bar(bar(C::kBarKFull + sn), ((u + 1) / NSK) & 1, abort_flag);
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
            }
            for (int t = 0; t < NQ; ++t) mma_commit(bar(C::kBarOFull + t), leader);
            mma_commit(bar(C::kBarMmaDone), leader);
            __syncwarp();
            drain_bar(bar(C::kBarMmaDone), 0);
        }
    } else {
        if constexpr (NQ == 2) setmaxnreg_inc<C::kRegsSoftmax>();
        // ------------------------------------------------------------ softmax
        const int t = warp >> 2;
        const int wq = warp & 3;
        const int rb = rb0 + t;
        const int row_local = wq * 32 + lane;
        const int row = rb * 128 + row_local;
        const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
        const uint32_t tS = tmem + lane_off + 128u * t;
        const uint32_t tO = tmem + lane_off + C::kOCol + D * t;
        const float cq = rb < p.nb ? p.scale_log2 * p.sq[static_cast<size_t>(bh) * p.nb + rb] : 0.0f;
        float m = -INFINITY, l = 0.f, l_r = 0.f;
        int cnt = 0;
        bool ok = true;
        for (int j = 0; j < nkb; ++j) {
            if (!((fwd8_flags<NQ>(p, rb0, j) >> t) & 1u)) continue;
            const float c = cq * p.sk[static_cast<size_t>(bh) * p.nb + j];   // score -> base-2 logit of this tile pair
            ok = wait_bar(bar(C::kBarSFull + t), cnt & 1, abort_flag);
            if (!ok) break;
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
            int hi = 127;
            if (p.causal && j == rb) hi = row_local;                          // diagonal tile
            if (j == p.nb - 1 && (p.N & 127)) hi = min(hi, (p.N & 127) - 1);  // key tail
            if (__any_sync(0xffffffffu, hi < 127)) {
#pragma unroll
                for (int k = 0; k < 128; ++k)
                    if (k > hi) sv[k] = -INFINITY;
            }
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
            const bool grow = m_cand > m + 8.0f;      // lazy rescale, as in the 16-bit forward (P <= 2^8 < 448)
            const float m_new = grow ? m_cand : m;
            const float alpha = grow ? ex2(m - m_new) : 1.0f;
            const float m_use = (m_new == -INFINITY) ? 0.0f : m_new;
            if (cnt > 0 && __any_sync(0xffffffffu, grow)) {
#pragma unroll 1
                for (int q = 0; q < D / 32; ++q) {
                    uint32_t o[32];
                    tmem_ld32_wait(tO + 32 * q, o);
#pragma unroll
                    for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
                    tmem_st32(tO + 32 * q, o);
                }
            }
            // P = 2^(s c - m) in fp32; P8 = E4M3(P), four codes per TMEM column
            float2 acc[4], acc_r[4];
#pragma unroll
            for (int a4 = 0; a4 < 4; ++a4) acc[a4] = acc_r[a4] = make_float2(0.f, 0.f);
            const float2 cc = make_float2(c, c), mm = make_float2(-m_use, -m_use);
            uint32_t p8[32];
#pragma unroll
            for (int g = 0; g < 32; ++g) {
                const float2 x0 = ffma2(make_float2(sv[4 * g], sv[4 * g + 1]), cc, mm);
                const float2 x1 = ffma2(make_float2(sv[4 * g + 2], sv[4 * g + 3]), cc, mm);
                const float2 e0 = make_float2(ex2(x0.x), ex2(x0.y));
                const float2 e1 = make_float2(ex2(x1.x), ex2(x1.y));
                const uint32_t lo = e4m3x2(e0.x, e0.y), hi2 = e4m3x2(e1.x, e1.y);
                p8[g] = lo | (hi2 << 16);
                acc[g & 3] = fadd2(acc[g & 3], fadd2(e0, e1));
                acc_r[g & 3] = fadd2(acc_r[g & 3], fadd2(e4m3x2_value(lo), e4m3x2_value(hi2)));
            }
            tmem_st32(tS, p8);
            const float2 s01 = fadd2(fadd2(acc[0], acc[1]), fadd2(acc[2], acc[3]));
            const float2 r01 = fadd2(fadd2(acc_r[0], acc_r[1]), fadd2(acc_r[2], acc_r[3]));
            l = l * alpha + (s01.x + s01.y);
            l_r = l_r * alpha + (r01.x + r01.y);
            m = m_new;
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(bar(C::kBarPFull + t));
            ++cnt;
        }
        if (ok && cnt > 0) ok = wait_bar(bar(C::kBarOFull + t), 0, abort_flag);
        tc_fence_after();
        // O_t (16-bit) staged in the finished K ring as 128-byte-swizzled
        // 64-column chunks, then written by TMA stores (rows >= N clipped)
        const bool epi = rb < p.nb && ok;
        uint8_t *stage = smem + C::kKOff + t * (D / 64) * C::kOChunk;
        if (epi) {
            const float sv_h = p.sv[static_cast<size_t>(bh) * p.nb];
            const float inv_l = (cnt > 0 && l_r > 0.f) ? sv_h / l_r : 0.0f;
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
                    pk[k] = pack2<BF16>(__uint_as_float(o[2 * k]) * inv_l, __uint_as_float(o[2 * k + 1]) * inv_l);
                uint8_t *srow = stage + (q >> 1) * C::kOChunk + row_local * 128;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int uu = (q & 1) * 4 + k;
                    *reinterpret_cast<uint4 *>(srow + ((uu ^ (row_local & 7)) << 4)) =
                        make_uint4(pk[4 * k], pk[4 * k + 1], pk[4 * k + 2], pk[4 * k + 3]);
                }
            }
            if (row < p.N)
                p.lse[static_cast<size_t>(bh) * p.N + row] =
                    (cnt > 0 && l > 0.f) ? (m + log2f(l)) * 0.69314718055994531f : -INFINITY;
        }
        fence_async_smem();
        named_sync(1 + t, 128);
        if (epi && wq == 0 && lane == 0) {
            for (int c = 0; c < D / 64; ++c)
                tma_store_3d(&tmo, smem_u32(stage + c * C::kOChunk), c * 64, rb * 128, bh);
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
