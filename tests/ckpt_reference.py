"""The scan's checkpoints for the host-emulation tests of the kernels that store or read them:
the oracle's states before every 16th step (oracle.selective_scan_ckpt on CrossScan(x)),
rearranged into the kernels' storage order."""
import numpy as np

from oracle import oracle as orc


def checkpoints(inp, B, D, L, N):
    """The state before every 16th step of each direction's sequence, (B, 4D, ceil(L/16), 16)
    fp32, in the kernels' order: state q + 2n at q*8 + n.  Softplus on."""
    xs = orc.cross_scan(inp["x"]).reshape(B, 4 * D, L)
    dts = inp["dts"].reshape(B, 4 * D, L)
    _, ck = orc.selective_scan_ckpt(xs, dts, inp["A_logs"], inp["Bs"], inp["Cs"], 16, Dv=inp["Ds"],
                                    delta_bias=inp["dt_bias"], delta_softplus=True)
    order = np.empty(N, dtype=int)
    for n in range(8):
        for q in range(2):
            order[q * 8 + n] = q + 2 * n
    return np.ascontiguousarray(ck[..., order].astype(np.float32))
