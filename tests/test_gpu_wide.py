"""GPU parity of dH_s and dW_s, element by element, at the hidden widths of
the pages' workloads.

The gradient kernel cuts H into 512-column tiles (two N = 256 halves per CTA
pair) and runs the H block as the fast tile index; these cases reach several
H blocks (H = 2048: 4, H = 4096: 8, H = 2560: 5), an H that is not a multiple
of 512 (1152: blocks of 512, 512, 128), more than one backward vocabulary
chunk with a ragged last tile, and several 256-row pair tiles of compacted
rows.  Every element of dH_s and dW_s is compared with the float64 oracle
(relative max-norm 2e-2 over the whole gradient and over every 512-column
H block separately, so that a block with small values cannot hide an error),
and the per-token loss within |dL| <= 1e-4 + 1e-3 |L|.
"""

import numpy as np
import pytest

from tests.gpu_cases import GRAD_RTOL, assert_tok_close, grad_rel_err, run_gpu, run_oracle, small_case, to_np

pytestmark = pytest.mark.gpu

CASES = [
    # B, Sm1, H, V, payload, mask, reduction
    (2, 300, 2048, 65536 + 4200, "hidden", "random", 1),   # 4 H blocks, 2 vocab chunks, ragged last tile
    (2, 150, 4096, 65536 + 1000, "hidden", "random", 2),   # 8 H blocks, 2 vocab chunks
    (1, 300, 1152, 3000, "hidden", "random", 1),           # H blocks 512, 512, 128
    (2, 700, 2048, 20000, "hidden", "random", 1),          # ~700 rows: 3 pair tiles of rows
    (1, 260, 2560, 5000, "hidden", "all", 2),              # N = 260: one row past a pair tile, 5 H blocks
    (2, 300, 2048, 8200, "logits", "random", 1),           # teacher-logits payload, 4 H blocks
]


def _block_errors(gpu, ref, width=512):
    g = gpu if isinstance(gpu, np.ndarray) else to_np(gpu)
    r = np.asarray(ref)
    out = []
    for c0 in range(0, r.shape[1], width):
        rb_ = r[:, c0:c0 + width]
        scale = np.max(np.abs(rb_))
        err = np.max(np.abs(g[:, c0:c0 + width] - rb_))
        out.append(err / scale if scale > 0 else err)
    return out


@pytest.mark.parametrize("B,Sm1,H,V,payload,mask,red", CASES)
def test_wide_hidden_elementwise(B, Sm1, H, V, payload, mask, red):
    inp = small_case(B=B, Sm1=Sm1, H=H, V=V, payload=payload, mask=mask, seed=H + V % 97)
    g = run_gpu(inp, red)
    r = run_oracle(inp, red)
    assert g["N"] == r["N"]
    assert_tok_close(g["loss_tok"], r["loss_tok"])
    assert abs(float(g["loss"]) - r["loss"]) <= 1e-4 + 1e-3 * abs(r["loss"])
    assert grad_rel_err(g["dH_s"], r["dH_s"]) < GRAD_RTOL
    assert grad_rel_err(g["dW_s"], r["dW_s"]) < GRAD_RTOL
    # every 512-column H block on its own scale
    assert max(_block_errors(g["dW_s"], r["dW_s"])) < GRAD_RTOL
    trainable = inp["mask"].numpy().reshape(-1) != 0
    assert max(_block_errors(to_np(g["dH_s"])[trainable], r["dH_s"][trainable])) < GRAD_RTOL
