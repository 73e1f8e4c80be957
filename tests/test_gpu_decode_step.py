"""pa_decode_step (the cache write and the attention of one decode step in one
call, the attention launched as a programmatic dependent of the write) on the GPU.

It must give exactly what pa_reshape_and_cache followed by pa_decode gives: the
caches bit for bit and the output bit for bit.  The rows of this step's new
tokens hold NaN before the call (gpu_cases poisons every row no stored token
uses), so an attention read that ran ahead of the write would put NaN into the
output.  The 13B case runs consecutive appending steps through the call and is
checked against the oracle as well.
"""
import numpy as np
import pytest
import torch

from gpu_cases import Step, assert_close, bits, device_inputs, oracle_decode, run_library
import oracle as oracle_pkg
from paged_kv_cache_374_b200 import binding as pa

pytestmark = pytest.mark.gpu


def _step_call(step, t, err=None, partition_tokens=0):
    tables, lens, slots = device_inputs(step, t)
    out = torch.empty_like(t["q"])
    pa.pa_decode_step(t["k"], t["v"], slots, t["q"], t["k_cache"], t["v_cache"], tables, lens, step.spec.scale,
                      step.spec.num_kv_heads, out, partition_tokens=partition_tokens, err_word=err)
    return out


@pytest.mark.parametrize("name,ptok", [("tiny", 0), ("llama7b", 0), ("gqa70b", 0), ("llama13b", 0),
                                       ("llama7b", 512)])
def test_decode_step_equals_write_then_decode(name, ptok):
    step = Step(name)
    t = step.tensors()
    t2 = {k: v.clone() for k, v in t.items()}
    # this step's slots hold NaN until the write
    slots = torch.from_numpy(step.slots).cuda()
    assert torch.isnan(t["k_cache"].view(-1, step.spec.num_kv_heads, step.spec.head_dim)[slots]).all()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = _step_call(step, t, err=err, partition_tokens=ptok)
    ref = run_library(step, t2, partition_tokens=ptok)
    torch.cuda.synchronize()
    assert err.item() == 0
    assert np.array_equal(bits(t["k_cache"]), bits(t2["k_cache"]))
    assert np.array_equal(bits(t["v_cache"]), bits(t2["v_cache"]))
    assert not torch.isnan(out).any()
    assert torch.equal(out, ref)


def test_decode_step_13b_appending_steps_against_the_oracle():
    """Six consecutive steps of the 13B workload through pa_decode_step: a1 on the
    host each step (new blocks at 16-token boundaries), then the one call; the
    oracle replays the cache writes and checks sampled pairs every step and every
    pair at the last."""
    step = Step("llama13b")
    t = step.tensors()
    kc_host, vc_host = bits(t["k_cache"]), bits(t["v_cache"])
    o = oracle_pkg.get()
    rng = np.random.default_rng(8)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(98)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    for i in range(6):
        if i > 0:
            step.slots = step.append()
            for key in ("q", "k", "v"):
                t[key] = torch.randn(t[key].shape, generator=gen, device="cuda").to(t[key].dtype)
        out = _step_call(step, t, err=err)
        torch.cuda.synchronize()
        o.reshape_and_cache(bits(t["k"]), bits(t["v"]), step.slots, kc_host, vc_host)
        q_host = bits(t["q"])
        if i == 5:
            assert np.array_equal(bits(t["k_cache"]), kc_host) and np.array_equal(bits(t["v_cache"]), vc_host)
            ref = oracle_decode(step, q_host, kc_host, vc_host)
            assert_close(out, ref, step.dtype, f"step {i}")
        else:
            pairs = np.array([(int(rng.integers(0, step.spec.num_seqs)), int(rng.integers(0, step.spec.num_heads)))
                              for _ in range(12)], dtype=np.int32)
            ref = oracle_decode(step, q_host, kc_host, vc_host, pairs=pairs)
            got = out[torch.from_numpy(pairs[:, 0]).long(), torch.from_numpy(pairs[:, 1]).long()]
            assert_close(got, ref, step.dtype, f"step {i}")
    assert err.item() == 0


def test_decode_step_checks_both_calls_first():
    """A bad argument of either half launches nothing: the cache stays untouched."""
    step = Step("tiny")
    t = step.tensors()
    before = bits(t["k_cache"]).copy()
    tables, lens, slots = device_inputs(step, t)
    out = torch.empty_like(t["q"])
    with pytest.raises(pa.PAError):      # workspace too small for the decode half
        pa.pa_decode_step(t["k"], t["v"], slots, t["q"], t["k_cache"], t["v_cache"], tables, lens, 0.125, 4, out,
                          workspace=torch.zeros(16, dtype=torch.uint8, device="cuda"))
    torch.cuda.synchronize()
    assert np.array_equal(bits(t["k_cache"]), before)


@pytest.mark.parametrize("name", ["llama7b", "gqa70b"])
def test_decode_step_fp8_equals_write_then_decode(name):
    """pa_decode_step_fp8 against pa_reshape_and_cache_fp8 followed by
    pa_decode_fp8: codes and output bit for bit (MHA and the tensor-core GQA
    policy)."""
    step = Step(name, num_seqs=8)
    t = step.tensors()
    to_codes = lambda x: (x.float() * 32).clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8)
    kc, vc = to_codes(t["k_cache"]), to_codes(t["v_cache"])
    kc2, vc2 = kc.clone(), vc.clone()
    tables, lens, slots = device_inputs(step, t)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.empty_like(t["q"])
    pa.pa_decode_step_fp8(t["k"], t["v"], slots, t["q"], kc, vc, tables, lens, step.spec.scale, 1 / 32, 1 / 32,
                          step.spec.num_kv_heads, out, err_word=err)
    pa.pa_reshape_and_cache_fp8(t["k"], t["v"], slots, kc2, vc2, 1 / 32, 1 / 32)
    ref = torch.empty_like(out)
    pa.pa_decode_fp8(t["q"], kc2, vc2, tables, lens, step.spec.scale, 1 / 32, 1 / 32, step.spec.num_kv_heads, ref)
    torch.cuda.synchronize()
    assert err.item() == 0
    assert torch.equal(kc, kc2) and torch.equal(vc, vc2)
    assert not torch.isnan(out).any()
    assert torch.equal(out, ref)
