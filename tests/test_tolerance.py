"""The parity tests' tolerance helper, checked on the CPU: half_ulp(ref) must be
exactly the largest error that rounding ref once to fp16 / bf16 can make (torch
does the rounding), so that "bound + half an ulp" allows the one final rounding
and nothing more."""
import numpy as np
import torch

from gpu_cases import half_ulp
from paged_kv_cache_374_b200 import workloads as wk


def test_half_ulp_is_the_rounding_bound():
    rng = np.random.default_rng(5)
    # fp32 values: the kernels round an fp32 result once (torch takes float64
    # through float32 first, which would round twice)
    x = np.concatenate([rng.normal(0, 1, 20000), rng.normal(0, 6, 20000),
                        rng.uniform(-300, 300, 20000)]).astype(np.float32).astype(np.float64)
    for dtype, tdt in ((wk.F16, torch.float16), (wk.BF16, torch.bfloat16)):
        r = torch.from_numpy(x).to(tdt).double().numpy()
        err, h = np.abs(r - x), half_ulp(x, dtype)
        assert np.all(err <= h * (1 + 1e-12))
        assert np.max(err / h) > 0.99            # reached: not a loose bound
    # the values the max-abs bounds meet: bf16 at |out| = 4, fp16 at |out| = 8
    assert half_ulp(np.array([4.0]), wk.BF16)[0] == 2.0 ** -6 > 1e-2
    assert half_ulp(np.array([3.99]), wk.BF16)[0] == 2.0 ** -7 < 1e-2
    assert half_ulp(np.array([8.0]), wk.F16)[0] == 2.0 ** -8 > 2e-3
