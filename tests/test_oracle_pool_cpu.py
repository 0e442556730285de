"""The chunked full-output comparison used by the large prefill parity tests,
checked on the CPU: the oracle's own output (rounded to bf16, as a kernel's
would be) passes, and a planted mistake in one row of one chunk is caught."""
import numpy as np
import torch

from compressed_sliding_window_b200 import inputs as I
from oracle import hca_oracle as O
from tests.oracle_pool import prefill_full_errors


def test_pool_matches_direct_oracle_and_catches_a_planted_error():
    cfg = I.PrefillConfig("pool_check", B=1, T=I.CHUNK + 300, seed=31, k_scale=0.5)
    x = I.prefill_inputs(cfg)
    f64 = lambda t: t.float().numpy().astype(np.float64)  # noqa: E731
    ref = O.prefill_forward(f64(x["q"]), f64(x["k"]), f64(x["v"]), f64(x["s"]), f64(x["g"]))
    out = torch.from_numpy(ref).to(torch.bfloat16)
    max_abs, rel, finite = prefill_full_errors(cfg, out, workers=2)
    assert finite and max_abs < 1e-2 and 0 < rel < 5e-3
    bad = out.clone()
    bad[0, I.CHUNK + 17, 5] += 0.25          # one row of the second (ragged) chunk
    max_abs2, rel2, _ = prefill_full_errors(cfg, bad, workers=2)
    assert max_abs2 > 0.2 and rel2 > rel
