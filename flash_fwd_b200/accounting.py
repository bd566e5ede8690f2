"""FLOP and byte accounting for exact attention (host arithmetic only).

* Forward FLOPs: two matrix products of 2*N*N*d each per (batch, head), so
  4*B*H*N^2*d, halved under the causal mask.
* Backward FLOPs: five matrix products against the forward's two, so 2.5x the
  forward ("FlashAttention 深度解析", section 四).
* Block-sparse: only kept 128 x 128 blocks count, 4*d*blk^2 per kept block per
  (batch, head) for the forward.
* General problems (query and key lengths that differ, sliding windows):
  4*d per visible (query, key) pair per (batch, head), the pairs counted
  exactly from the visibility band (bottom-right aligned).
* Minimum HBM bytes of the fused forward: read Q, K, V, write O (4*N*d*e) plus
  one fp32 LSE per row; of the backward: read Q, K, V, O, dO, LSE, D and write
  dQ, dK, dV (8*N*d*e + 8*N), before the fp32 dQ accumulator this design adds.
* The worked case study of "FlashAttention原理概览" section 3.4 (S bytes, Q/K/V
  read bytes, O write bytes, S traffic when S is materialised) and the SRAM
  budget of its section 3.1 are reproduced by the helpers below.
"""


def fwd_flops(B, H, N, d, causal=False):
    f = 4.0 * B * H * N * N * d
    return f / 2 if causal else f


def bwd_flops(B, H, N, d, causal=False):
    return 2.5 * fwd_flops(B, H, N, d, causal)


def sparse_fwd_flops(B, H, d, kept_blocks, blk=128):
    return 4.0 * B * H * d * blk * blk * kept_blocks


def sparse_bwd_flops(B, H, d, kept_blocks, blk=128):
    return 2.5 * sparse_fwd_flops(B, H, d, kept_blocks, blk)


def fwd_min_bytes(B, H, N, d, elem=2):
    return B * H * (4 * N * d * elem + 4 * N)


def bwd_min_bytes(B, H, N, d, elem=2):
    return B * H * (8 * N * d * elem + 8 * N)


def s_matrix_bytes(B, H, N, elem=2):
    """Bytes of one materialised N x N score matrix over all heads."""
    return B * H * N * N * elem


def standard_s_traffic(B, H, N, elem=2):
    """S written once and read three times by the unfused method."""
    return 4 * s_matrix_bytes(B, H, N, elem)


def qkv_read_bytes(N, d, elem=2):
    return 3 * N * d * elem


def o_write_bytes(N, d, elem=2):
    return N * d * elem


def sram_tile_bytes(Br, Bc, d, elem):
    """Q block + K/V block + S block, the budget Br*d + Bc*d + Br*Bc <= M."""
    return (Br * d + Bc * d + Br * Bc) * elem


def io_bound_elems(N, d, M):
    """The Theta(N^2 d^2 / M) HBM accesses of the tiled method (深度解析 section 三)."""
    return N * N * d * d / M


def visible_pairs(Nq, Nk, causal=False, window=None):
    """Number of (query, key) pairs a head attends to: query i sees keys
    i + Nk - Nq - left .. i + Nk - Nq + right (right = 0 under causal; a
    negative side is unbounded), clipped to 0 .. Nk - 1."""
    import numpy as np
    off = Nk - Nq
    left, right = (-1, -1) if window is None else window
    i = np.arange(Nq, dtype=np.int64)
    lo = np.zeros(Nq, dtype=np.int64) if left < 0 else np.maximum(i + off - left, 0)
    hi = np.full(Nq, Nk - 1, dtype=np.int64) if right < 0 else np.minimum(i + off + right, Nk - 1)
    if causal:
        hi = np.minimum(hi, i + off)
    return int(np.maximum(hi - lo + 1, 0).sum())


def general_fwd_flops(B, H, Nq, Nk, d, causal=False, window=None):
    return 4.0 * B * H * d * visible_pairs(Nq, Nk, causal, window)

