"""The scan's checkpoints in fp64, for the host-emulation tests of the kernels that store or read them."""
import numpy as np

from oracle import oracle as orc


def checkpoints(inp, B, D, L, N):
    """The state before every 16th step of each direction's sequence, (B, 4D, ceil(L/16), 16)
    fp32, in the kernels' order: state q + 2n at q*8 + n.  The forward recurrence of the core
    in fp64 on CrossScan(x), softplus on, from the oracle's cross_scan."""
    xs = orc.cross_scan(inp["x"])
    z = inp["dts"].astype(np.float64) + inp["dt_bias"].reshape(4, D)[None, :, :, None]
    delta = np.where(z > 0, z + np.log1p(np.exp(-np.abs(z))), np.log1p(np.exp(z)))
    A = -np.exp(inp["A_logs"].astype(np.float64)).reshape(4, D, N)
    Bm = inp["Bs"].astype(np.float64)
    nck = (L + 15) // 16
    ck = np.zeros((B, 4, D, nck, N))
    h = np.zeros((B, 4, D, N))
    for l in range(L):
        if l % 16 == 0:
            ck[:, :, :, l // 16] = h
        h = np.exp(delta[..., l][..., None] * A[None]) * h + (delta[..., l] * xs[..., l])[..., None] * Bm[:, :, None, :, l]
    order = np.empty(N, dtype=int)
    for n in range(8):
        for q in range(2):
            order[q * 8 + n] = q + 2 * n
    return np.ascontiguousarray(ck[..., order].reshape(B, 4 * D, nck, N).astype(np.float32))
