"""GPU parity at the size limits of the chunk scan's indexing.

One sequence of 2^21 + 37 tokens and 16 heads: x and y hold more than 2^31 elements, so every
flat index into them needs 64 bits, and each (sequence, head) unit spans about nine CTAs.  The
state therefore crosses a chain of CTA hand-offs before it reaches the unit's end.  The oracle
runs two sampled heads whole.
"""
import numpy as np
import pytest
import torch

import oracle
from quantized_mamba_ssd_b200 import build as qbuild
from quantized_mamba_ssd_b200 import ssd_i8
from parity_util import check_close, check_i8

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    qbuild.build()
    ssd_i8.library()


def test_more_than_2_pow_31_output_elements():
    L, H, P, N, G, Q = (1 << 21) + 37, 16, 64, 16, 1, 256
    assert L * H * P > 2 ** 31
    rng = np.random.default_rng(2024)
    # int8 codes drawn directly (the float activations of this size would not fit the host)
    x = rng.integers(-127, 128, size=(1, L, H, P), dtype=np.int8)
    B = rng.integers(-127, 128, size=(1, L, G, N), dtype=np.int8)
    C = rng.integers(-127, 128, size=(1, L, G, N), dtype=np.int8)
    dt = np.log1p(np.exp(rng.normal(-2.0, 0.5, size=(1, L, H)))).astype(np.float32)
    A = (-np.exp(rng.uniform(0.0, np.log(16.0), size=H))).astype(np.float32)
    D = rng.standard_normal(H).astype(np.float32)
    sx = rng.uniform(0.005, 0.02, size=H).astype(np.float32)
    sb = np.full(G, 0.01, dtype=np.float32)
    sc = np.full(G, 0.01, dtype=np.float32)
    heads = [0, H - 1]
    refs = {}
    for h in heads:
        yr, fr, _ = oracle.scan(x[:, :, h:h + 1], B, C, dt[:, :, h:h + 1], A[h:h + 1], D[h:h + 1],
                                sx[h:h + 1], sb, sc)
        refs[h] = (yr[0, :, 0, :], fr[0, 0])
    s_y = float(max(np.abs(r[0]).max() for r in refs.values()) / 127.0)
    fs = torch.empty((1, H, P, N), dtype=torch.float32, device=DEV)
    ws = torch.empty(ssd_i8.ssd_i8_chunk_scan_workspace_size(1, L, H, P, N, G, Q),
                     dtype=torch.uint8, device=DEV)
    y = ssd_i8.ssd_i8_chunk_scan(torch.from_numpy(x).to(DEV), torch.from_numpy(B).to(DEV),
                                 torch.from_numpy(C).to(DEV), torch.from_numpy(dt).to(DEV),
                                 torch.from_numpy(A).to(DEV), torch.from_numpy(D).to(DEV),
                                 torch.from_numpy(sx).to(DEV), torch.from_numpy(sb).to(DEV),
                                 torch.from_numpy(sc).to(DEV), Q, final_state=fs, y_dtype="i8",
                                 y_scale=s_y, workspace=ws)
    torch.cuda.synchronize()
    ssd_i8.ssd_i8_chunk_scan_status(ws)  # raises if a hand-off wait ran out along the chain
    for h in heads:
        yr, fr = refs[h]
        check_i8(y[0, :, h, :].cpu().numpy(), oracle.requant(yr, s_y))
        check_close(fs[0, h].cpu().numpy(), fr, f"final state of head {h}")
    # the last tokens of the last head sit past element 2^31 of y
    last = y[0, -3:, H - 1, :].cpu().numpy()
    check_i8(last, oracle.requant(refs[H - 1][0][-3:], s_y))
