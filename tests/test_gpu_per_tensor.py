"""Per-tensor (state-dict) FP8 conversion on the GPU vs the CPU oracle:
bit-exact codes and scales, both formats."""
import numpy as np
import pytest
import torch

import oracle
import synth
from conftest import to_device_bf16

pytestmark = pytest.mark.gpu

fp8 = pytest.importorskip("dit_rowwise_amax_b200")


def convert_and_check(arrays, fmt):
    dev = [to_device_bf16(a) for a in arrays]
    outs, scales = fp8.quantize_per_tensor(dev, fmt)
    torch.cuda.synchronize()
    s = scales.cpu().numpy()
    for i, a in enumerate(arrays):
        if a.size == 0:
            continue
        qo, so = oracle.quantize_tensor(a, fmt)
        assert np.float32(so).view(np.uint32) == s[i].view(np.uint32), f"scale {i}"
        q = outs[i].cpu().numpy()
        bad = np.argwhere(q.reshape(-1) != qo.reshape(-1))
        assert bad.size == 0, f"tensor {i}: {bad.size} codes differ, first {bad[:5].ravel().tolist()}"


@pytest.mark.parametrize("fmt", [oracle.E4M3FN, oracle.E5M2])
def test_small_mixed_set(fmt):
    arrays = [
        synth.state_dict_tensor("gpu/pt/a", (64, 96)),
        synth.state_dict_tensor("gpu/pt/b", (1000, 33)),       # numel not a multiple of 8
        np.zeros((17,), dtype=np.uint16),                       # all zero -> S = 1
        synth.state_dict_tensor("gpu/pt/c", (70000,)),          # spans several chunks, ragged end
        synth.state_dict_tensor("gpu/pt/d", (3,)),
        np.zeros((0,), dtype=np.uint16),                        # empty: skipped
        synth.state_dict_tensor("gpu/pt/e", (2048, 2048)),
    ]
    convert_and_check(arrays, fmt)


def test_many_tensors_cross_batches():
    arrays = [synth.state_dict_tensor(f"gpu/pt/many{i}", (8 * (i % 37 + 1),)) for i in range(450)]
    convert_and_check(arrays, oracle.E4M3FN)


@pytest.mark.slow
@pytest.mark.parametrize("fmt", [oracle.E4M3FN, oracle.E5M2])
def test_full_state_dict(fmt):
    """The 32-block synthetic DiT weight set (192 tensors, 1.61e9 elements)."""
    layout = synth.state_dict_layout()
    host = [synth.state_dict_tensor(n, s) for n, s in layout]
    dev = [to_device_bf16(a) for a in host]
    outs, scales = fp8.quantize_per_tensor(dev, fmt)
    torch.cuda.synchronize()
    s = scales.cpu().numpy()
    for i, a in enumerate(host):
        qo, so = oracle.quantize_tensor(a, fmt)
        assert np.float32(so).view(np.uint32) == s[i].view(np.uint32), layout[i][0]
        assert np.array_equal(outs[i].cpu().numpy(), qo), layout[i][0]
        outs[i] = None
        dev[i] = None


def test_convert_state_dict_contract():
    sd = {
        "w1": to_device_bf16(synth.state_dict_tensor("gpu/sd/w1", (128, 64))),
        "w2": to_device_bf16(synth.state_dict_tensor("gpu/sd/w2", (256,))),
        "step": torch.tensor(3),
        "f32": torch.ones(4, device="cuda"),
        "idx": torch.arange(5, device="cuda"),
        "done": torch.zeros(2, device="cuda").to(torch.float8_e5m2),
    }
    out, scales = fp8.convert_state_dict(sd)  # default float8_e5m2
    assert out["w1"].dtype == torch.float8_e5m2 and out["w2"].dtype == torch.float8_e5m2
    assert out["f32"].dtype == torch.float8_e5m2  # floating tensors of every supported dtype convert
    assert out["step"] is sd["step"] and out["idx"] is sd["idx"] and out["done"] is sd["done"]
    assert set(scales) == {"w1", "w2", "f32"}
    qo, so = oracle.quantize_tensor(synth.state_dict_tensor("gpu/sd/w1", (128, 64)), oracle.E5M2)
    assert np.array_equal(out["w1"].view(torch.uint8).cpu().numpy(), qo)
    assert float(scales["w1"]) == so
    with pytest.raises(ValueError, match="not convertible"):
        fp8.convert_state_dict({"w": torch.ones(4, dtype=torch.float64, device="cuda")})
    with pytest.raises(ValueError, match="CUDA device"):
        fp8.convert_state_dict({"w": torch.ones(4, dtype=torch.float16)})
    with pytest.raises(ValueError, match="Invalid input"):
        fp8.convert_state_dict({})
    with pytest.raises(ValueError, match="Invalid input"):
        fp8.convert_state_dict([1, 2])
    with pytest.raises(fp8.Fp8DitError, match="No tensor converted"):
        fp8.convert_state_dict({"a": torch.zeros(3, dtype=torch.bfloat16, device="cuda")[:0]})


def test_empty_set_is_an_error():
    with pytest.raises(fp8.Fp8DitError) as e:
        fp8.quantize_per_tensor([torch.zeros(0, dtype=torch.bfloat16, device="cuda")], fp8.E4M3FN)
    assert e.value.status == 3


def f16_f32_arrays():
    """A mixed bf16 / fp16 / fp32 weight set: ragged sizes (tails of the 8- and
    4-element vectors), several chunks, subnormals, an all-zero tensor, and
    values that are not exact in bf16."""
    rng = np.random.default_rng(11)
    out = []
    for i, n in enumerate((64 * 96, 1000 * 33, 70001, 3, 17, 2048 * 2048 + 5)):
        w = rng.standard_normal(n) * 0.02
        w[rng.integers(0, n, max(1, n // 1000))] *= 50
        if i % 3 == 0:
            out.append(("bf16", synth.state_dict_tensor(f"gpu/pt/mix{i}", (n,))))
        elif i % 3 == 1:
            out.append(("f16", w.astype(np.float16)))
        else:
            out.append(("f32", w.astype(np.float32)))
    out.append(("f16", (np.arange(1, 4001, dtype=np.float64) * 2.0 ** -24).astype(np.float16)))  # fp16 subnormals
    out.append(("f32", np.zeros(9, dtype=np.float32)))
    out.append(("f32", (rng.standard_normal(5000) * 1e-38).astype(np.float32)))  # tiny amax: subnormal S
    return out


def to_device(kind, a):
    return to_device_bf16(a) if kind == "bf16" else torch.from_numpy(a).cuda()


@pytest.mark.parametrize("fmt", [oracle.E4M3FN, oracle.E5M2])
def test_mixed_dtypes_bit_exact(fmt):
    arrays = f16_f32_arrays()
    outs, scales = fp8.quantize_per_tensor([to_device(k, a) for k, a in arrays], fmt)
    torch.cuda.synchronize()
    s = scales.cpu().numpy()
    for i, (kind, a) in enumerate(arrays):
        qo, so = oracle.quantize_tensor_typed(a, fmt)
        assert np.float32(so).view(np.uint32) == s[i].view(np.uint32), f"scale {i} ({kind})"
        q = outs[i].cpu().numpy()
        bad = np.flatnonzero(q != qo)
        assert bad.size == 0, f"tensor {i} ({kind}): {bad.size} codes differ, first {bad[:5].tolist()}"


def test_convert_state_dict_mixed_dtypes():
    """A state-dict of bf16, fp16 and fp32 weights converts in one call, every
    tensor bit-exact against the oracle."""
    arrays = f16_f32_arrays()
    sd = {f"t{i}": to_device(k, a) for i, (k, a) in enumerate(arrays)}
    out, scales = fp8.convert_state_dict(sd, "float8_e4m3fn")
    for i, (kind, a) in enumerate(arrays):
        qo, so = oracle.quantize_tensor_typed(a, oracle.E4M3FN)
        assert out[f"t{i}"].dtype == torch.float8_e4m3fn
        assert np.array_equal(out[f"t{i}"].view(torch.uint8).cpu().numpy(), qo), f"t{i} ({kind})"
        assert np.float32(float(scales[f"t{i}"])) == np.float32(so)
