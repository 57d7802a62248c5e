"""Independent fp64 forms of the SSD layer, used only to pin the sequential oracle.

TEST INFRASTRUCTURE ONLY; written separately from ``ssd_oracle.c`` and sharing
nothing with it or with the CUDA library.

Source: "Compiler-First State Space Duality and Portable O(1) Autoregressive
Caching for Inference", section "2. Metodologia": the recurrence is chunkable
(fixed-size chunks), its intra-chunk part is a masked matrix product built with
a static lower-triangular mask, and the decay exponent is taken in fp32 or
wider.  Both functions below restate that structure in numpy:

* ``chunked``: the chunked algorithm step by step --
  (1) per chunk, the inclusive cumulative sum ``Lam`` of ``dt * A_h``;
  (2) the intra-chunk output ``(L o C B^T) (dt x)`` with
      ``L[t, s] = exp(Lam_t - Lam_s)`` for ``s <= t`` and 0 otherwise;
  (3) the chunk's own end state from zero,
      ``sum_s exp(Lam_end - Lam_s) dt_s B_s x_s^T``, and the state carried
      across chunks, ``H_next = exp(Lam_end) H + s_chunk``;
  (4) the carried state's contribution to the outputs,
      ``exp(Lam_t) C_t^T H_chunk_start``, plus the skip ``D_h x_t``.
* ``quadratic``: the whole sequence as one masked matrix,
  ``y = (L o C B^T)(dt x) + D x`` with ``L`` over all T tokens
  (exact only while the decay products stay representable -- tiny inputs).

Layouts are the same as the oracle's: inputs as in the C ABI, outputs
``y`` [b][T][H][P] and ``state`` [b][H][P][N].
"""
from __future__ import annotations

import numpy as np


def _prep(x, dt, A, B, C, D):
    x = np.asarray(x, dtype=np.float64)
    dt = np.asarray(dt, dtype=np.float64)
    A = np.asarray(A, dtype=np.float64)
    B = np.asarray(B, dtype=np.float64)
    C = np.asarray(C, dtype=np.float64)
    D = np.asarray(D, dtype=np.float64)
    b, T, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    hg = H // G
    # expand groups to heads: head h reads group h // (H / G)
    Bh = np.repeat(B, hg, axis=2)  # [b][T][H][N]
    Ch = np.repeat(C, hg, axis=2)
    return x, dt, A, Bh, Ch, D


def chunked(x, dt, A, B, C, D, chunk_len, init=None):
    x, dt, A, Bh, Ch, D = _prep(x, dt, A, B, C, D)
    b, T, H, P = x.shape
    N = Bh.shape[3]
    y = np.zeros((b, T, H, P))
    Hst = np.zeros((b, H, N, P)) if init is None else \
        np.asarray(init, dtype=np.float64).reshape(b, H, P, N).transpose(0, 1, 3, 2).copy()
    for c0 in range(0, T, chunk_len):
        c1 = min(c0 + chunk_len, T)
        q = c1 - c0
        xc = x[:, c0:c1]                      # [b][q][H][P]
        dtc = dt[:, c0:c1]                    # [b][q][H]
        Bc = Bh[:, c0:c1]                     # [b][q][H][N]
        Cc = Ch[:, c0:c1]
        # (1) inclusive cumsum of dt*A within the chunk
        lam = np.cumsum(dtc * A[None, None, :], axis=1)          # [b][q][H]
        # (2) intra-chunk masked product
        seg = lam[:, :, None, :] - lam[:, None, :, :]            # [b][t][s][H]
        tril = np.tril(np.ones((q, q), dtype=bool))
        L = np.where(tril[None, :, :, None], np.exp(np.where(tril[None, :, :, None], seg, 0.0)), 0.0)
        CB = np.einsum("bthn,bshn->btsh", Cc, Bc)
        Pm = CB * L * dtc[:, None, :, :]                         # [b][t][s][H]
        y_diag = np.einsum("btsh,bshp->bthp", Pm, xc)
        # (4) contribution of the state carried into this chunk
        y_off = np.einsum("bthn,bhnp->bthp", Cc, Hst) * np.exp(lam)[..., None]
        y[:, c0:c1] = y_diag + y_off + D[None, None, :, None] * xc
        # (3) chunk end state and the carry
        w = np.exp(lam[:, -1:, :] - lam) * dtc                   # [b][q][H]
        s_chunk = np.einsum("bshn,bsh,bshp->bhnp", Bc, w, xc)
        Hst = np.exp(lam[:, -1, :])[..., None, None] * Hst + s_chunk
    return y, Hst.transpose(0, 1, 3, 2).copy()


def quadratic(x, dt, A, B, C, D):
    """Whole-sequence masked form (no carried state); tiny inputs only."""
    x, dt, A, Bh, Ch, D = _prep(x, dt, A, B, C, D)
    b, T, H, P = x.shape
    y = np.zeros((b, T, H, P))
    tril = np.tril(np.ones((T, T), dtype=bool))
    for bi in range(b):
        for h in range(H):
            dA = dt[bi, :, h] * A[h]
            # L[t, s] = prod_{r=s+1..t} exp(dA_r), formed from explicit products
            L = np.zeros((T, T))
            for t in range(T):
                acc = 1.0
                L[t, t] = 1.0
                for s in range(t - 1, -1, -1):
                    acc *= np.exp(dA[s + 1])
                    L[t, s] = acc
            M = (Ch[bi, :, h, :] @ Bh[bi, :, h, :].T) * L * tril
            y[bi, :, h, :] = M @ (dt[bi, :, h, None] * x[bi, :, h, :]) + D[h] * x[bi, :, h, :]
    return y
