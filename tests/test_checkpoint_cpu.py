"""Quantized checkpoints in ordinary safetensors files (the int4 and int8
cards use the standard container, nothing of their own), read by the
library's rt_st_* calls with the format detected from the tensor dtypes.  Files are written here by the independent
`safetensors` package from tensors the library's own quantizers produce; the
reader must return the same bytes and the right format and sizes, and refuse
malformed files."""
import json
import struct

import numpy as np
import pytest

import int8_dequant_gemm_b200 as rtq
from int8_dequant_gemm_b200 import build as rtq_build
from int8_dequant_gemm_b200 import workloads as wl

torch = pytest.importorskip("torch")
st = pytest.importorskip("safetensors.torch")


@pytest.fixture(scope="module", autouse=True)
def built():
    rtq_build.build()
    return rtq.lib()


def _quantized():
    Wa = wl.weights(256, 512, 1)
    Wb = wl.weights(128, 1024, 2)
    Wc = wl.weights(64, 256, 3)
    q4 = rtq.quantize_q4_g32(Wa)
    q8 = rtq.quantize_q8_row(Wb)
    f8 = rtq.quantize_e4m3(Wc)
    return q4, q8, f8


def _write(path, q4, q8, f8, q4_scale_2d=False, q8_scale_2d=False):
    sm = q4[1].reshape(q4[1].shape[0], -1) if q4_scale_2d else q4[1]
    sc = q8[1].reshape(-1, 1) if q8_scale_2d else q8[1]
    tensors = {
        "blocks.0.attn.wq": torch.from_numpy(q4[0]),
        "blocks.0.attn.wq.q4_scale": torch.from_numpy(sm.view(np.float16)),
        "blocks.0.ffn.w2": torch.from_numpy(q8[0]),
        "blocks.0.ffn.w2.q_scale": torch.from_numpy(sc),
        "blocks.0.attn.wo": torch.from_numpy(f8).view(torch.float8_e4m3fn),
        "blocks.0.norm.bias": torch.zeros(512, dtype=torch.float32),
    }
    st.save_file(tensors, str(path), metadata={"quantization": "mixed"})


@pytest.mark.parametrize("variant", [(False, False), (True, True)])
def test_formats_detected_and_bytes_returned(tmp_path, variant):
    q4, q8, f8 = _quantized()
    p = tmp_path / "model.q.safetensors"
    _write(p, q4, q8, f8, *variant)
    with rtq.Checkpoint(p) as ck:
        assert len(ck) == 6
        fmt, codes, sm = ck.weight("blocks.0.attn.wq")
        assert fmt == rtq.FMT_Q4 and np.array_equal(codes, q4[0]) and np.array_equal(sm, q4[1])
        fmt, codes, sc = ck.weight("blocks.0.ffn.w2")
        assert fmt == rtq.FMT_Q8 and np.array_equal(codes, q8[0]) and np.array_equal(sc, q8[1])
        fmt, codes, none = ck.weight("blocks.0.attn.wo")
        assert fmt == rtq.FMT_E4M3 and np.array_equal(codes, f8) and none is None
        for name, status in (("nope", 13), ("blocks.0.norm.bias", 3)):
            with pytest.raises(rtq.RtqError) as e:
                ck.weight(name)
            assert e.value.status == status


def _raw(header: dict, data: bytes, pad=0):
    h = json.dumps(header).encode() + b" " * pad
    return struct.pack("<Q", len(h)) + h + data


def test_malformed_files_are_refused(tmp_path):
    good = {"w": {"dtype": "I8", "shape": [2, 16], "data_offsets": [0, 32]},
            "w.q_scale": {"dtype": "F32", "shape": [2], "data_offsets": [32, 40]}}
    cases = {
        "ok": (_raw(good, bytes(40)), 0),
        "truncated_header": (struct.pack("<Q", 1000) + b"{}", 12),
        "tiny": (b"abc", 12),
        "bad_json": (struct.pack("<Q", 5) + b"{\"w\":", 12),
        "offset_past_end": (_raw(good, bytes(39)), 12),
        "size_mismatch": (_raw({"w": {"dtype": "I8", "shape": [2, 16],
                                       "data_offsets": [0, 31]}}, bytes(40)), 12),
        "unknown_dtype": (_raw({"w": {"dtype": "Q3", "shape": [1],
                                       "data_offsets": [0, 1]}}, bytes(1)), 12),
        "trailing_garbage": (struct.pack("<Q", 4) + b"{}xx", 12),
    }
    for name, (blob, status) in cases.items():
        p = tmp_path / f"{name}.safetensors"
        p.write_bytes(blob)
        if status == 0:
            with rtq.Checkpoint(p) as ck:
                assert ck.weight("w")[0] == rtq.FMT_Q8
            continue
        with pytest.raises(rtq.RtqError) as e:
            rtq.Checkpoint(p)
        assert e.value.status == status, name
    with pytest.raises(rtq.RtqError) as e:
        rtq.Checkpoint(tmp_path / "missing.safetensors")
    assert e.value.status == 11


def test_companion_mismatches(tmp_path):
    bad = {
        # q4 companion with the wrong dtype
        "q4_dtype": {"w": {"dtype": "U8", "shape": [2, 16], "data_offsets": [0, 32]},
                     "w.q4_scale": {"dtype": "F32", "shape": [2, 1, 2], "data_offsets": [32, 48]}},
        # q4 companion with the wrong group count
        "q4_shape": {"w": {"dtype": "U8", "shape": [2, 16], "data_offsets": [0, 32]},
                     "w.q4_scale": {"dtype": "F16", "shape": [2, 2, 2], "data_offsets": [32, 48]}},
        # q8 scale of the wrong length
        "q8_len": {"w": {"dtype": "I8", "shape": [2, 16], "data_offsets": [0, 32]},
                   "w.q_scale": {"dtype": "F32", "shape": [3], "data_offsets": [32, 44]}},
    }
    for name, header in bad.items():
        end = max(v["data_offsets"][1] for v in header.values())
        p = tmp_path / f"{name}.safetensors"
        p.write_bytes(_raw(header, bytes(end)))
        with rtq.Checkpoint(p) as ck:
            with pytest.raises(rtq.RtqError) as e:
                ck.weight("w")
            assert e.value.status == 12, name
    # a q8 weight without its companion
    p = tmp_path / "lonely.safetensors"
    p.write_bytes(_raw({"w": {"dtype": "I8", "shape": [2, 16], "data_offsets": [0, 32]}}, bytes(32)))
    with rtq.Checkpoint(p) as ck:
        with pytest.raises(rtq.RtqError) as e:
            ck.weight("w")
        assert e.value.status == 13
