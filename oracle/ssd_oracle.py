"""fp64 CPU oracle for the Mamba-2 state-space-duality (SSD) form -- TEST INFRASTRUCTURE.

Only the test suite may import this module; it shares nothing with the CUDA
path (no SSD kernel exists yet: this oracle comes first).

What it computes, in the quadratic (attention-like) form the pages give
("Mamba & Mamba-2 Architecture", section 3, "Mamba-2 and State Space Duality"):
the transition is a scalar per head, a_t = exp(delta_t * A_h), so the whole
sequence map is one 1-semiseparable matrix,

    Y = (M o (C Bbar^T)) X,     M[t, s] = prod_{k = s+1 .. t} a_k  (s <= t), 0 (s > t),

with query C, key Bbar, value X (the page's mapping to masked linear
attention).  Readings where the page's formulas were lost: Bbar_s = delta_s B_s
(the Euler input term the other pages use for the selective scan), B and C
shared by all heads ([B, L, N], one group), head dimension P, and an optional
initial state h0 [B, H, N, P] entering as C_t . (prod_{k <= t} a_k) h0.  The
final state is h_L = sum_s (prod_{k > s} a_k) Bbar_s x_s^T + (prod a) h0.

Every (batch, head) pair builds its L x L matrix explicitly (O(L^2)), so this
is for small sizes.
"""
from __future__ import annotations

import numpy as np


def ssd_matrix(delta_bh, A_h, B_b, C_b):
    """The L x L matrix M o (C Bbar^T) of one (batch, head): entry (t, s) =
    (C_t . B_s) * delta_s * prod_{k=s+1..t} exp(delta_k A_h) for s <= t, else 0."""
    delta_bh = np.asarray(delta_bh, np.float64)
    L = delta_bh.shape[0]
    a = np.exp(delta_bh * float(A_h))
    M = np.zeros((L, L))
    for t in range(L):
        p = 1.0
        for s in range(t, -1, -1):  # p = prod_{k=s+1..t} a_k
            M[t, s] = p
            p *= a[s]
    G = np.asarray(C_b, np.float64) @ np.asarray(B_b, np.float64).T  # (C_t . B_s)
    return M * G * delta_bh[None, :]


def ssd_forward(x, delta, A, B, C, h0=None):
    """SSD forward in fp64.

    x: [Bt, L, H, P]; delta: [Bt, L, H]; A: [H]; B, C: [Bt, L, N];
    h0: [Bt, H, N, P] or None.  Returns (y [Bt, L, H, P], h_final [Bt, H, N, P]).
    """
    x = np.asarray(x, np.float64)
    delta = np.asarray(delta, np.float64)
    A = np.asarray(A, np.float64)
    B = np.asarray(B, np.float64)
    C = np.asarray(C, np.float64)
    Bt, L, H, P = x.shape
    N = B.shape[2]
    y = np.zeros((Bt, L, H, P))
    hf = np.zeros((Bt, H, N, P))
    for b in range(Bt):
        for h in range(H):
            W = ssd_matrix(delta[b, :, h], A[h], B[b], C[b])
            y[b, :, h, :] = W @ x[b, :, h, :]
            a = np.exp(delta[b, :, h] * A[h])
            tail = np.ones(L)  # tail[s] = prod_{k=s+1..L-1} a_k
            for s in range(L - 2, -1, -1):
                tail[s] = tail[s + 1] * a[s + 1]
            hf[b, h] = (B[b] * (delta[b, :, h] * tail)[:, None]).T @ x[b, :, h, :]
            if h0 is not None:
                h0bh = np.asarray(h0, np.float64)[b, h]
                head = np.cumprod(a)  # prod_{k=0..t} a_k
                y[b, :, h, :] += (C[b] * head[:, None]) @ h0bh
                hf[b, h] += head[-1] * h0bh if L > 0 else h0bh
    return y, hf


def ssd_forward_chunked(x, delta, A, B, C, h0=None, block=64):
    """The same map computed the way the page's kernel organises it ("Mamba & Mamba-2
    Architecture", section 3: the sequence cut into blocks, e.g. 64 tokens): per block,
    the intra-block part (M_blk o C_blk Bbar_blk^T) X_blk, the block's own end state
    S = sum_s (prod_{k>s in block} a_k) Bbar_s x_s^T, and the state passed in from the
    earlier blocks, h <- (prod over the block of a) h + S, which reaches the block's
    outputs as C_t (prod_{k = block start .. t} a_k) h_in.  Same shapes as ssd_forward."""
    x = np.asarray(x, np.float64)
    delta = np.asarray(delta, np.float64)
    A = np.asarray(A, np.float64)
    B = np.asarray(B, np.float64)
    C = np.asarray(C, np.float64)
    Bt, L, H, P = x.shape
    N = B.shape[2]
    y = np.zeros((Bt, L, H, P))
    hf = np.zeros((Bt, H, N, P))
    for b in range(Bt):
        for h in range(H):
            state = np.zeros((N, P)) if h0 is None else np.asarray(h0, np.float64)[b, h].copy()
            for t0 in range(0, L, block):
                t1 = min(L, t0 + block)
                dl = delta[b, t0:t1, h]
                a = np.exp(dl * A[h])
                xb = x[b, t0:t1, h, :]
                # intra-block: the block's own semiseparable matrix
                y[b, t0:t1, h, :] = ssd_matrix(dl, A[h], B[b, t0:t1], C[b, t0:t1]) @ xb
                # inter-block: the carried-in state, decayed to each position of the block
                head = np.cumprod(a)
                y[b, t0:t1, h, :] += (C[b, t0:t1] * head[:, None]) @ state
                # the block's own end state, then the state passing
                tail = np.ones(t1 - t0)
                for s in range(t1 - t0 - 2, -1, -1):
                    tail[s] = tail[s + 1] * a[s + 1]
                S_blk = (B[b, t0:t1] * (dl * tail)[:, None]).T @ xb
                state = head[-1] * state + S_blk
            hf[b, h] = state
    return y, hf
