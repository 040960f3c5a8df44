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
    }
    out, scales = fp8.convert_state_dict(sd)  # default float8_e5m2
    assert out["w1"].dtype == torch.float8_e5m2 and out["w2"].dtype == torch.float8_e5m2
    assert out["step"] is sd["step"] and out["f32"] is sd["f32"]
    qo, so = oracle.quantize_tensor(synth.state_dict_tensor("gpu/sd/w1", (128, 64)), oracle.E5M2)
    assert np.array_equal(out["w1"].view(torch.uint8).cpu().numpy(), qo)
    assert float(scales["w1"]) == so
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
