"""A quantized checkpoint from file to GEMM: weights quantized by the oracle,
written with the independent `safetensors` package, read back through the
library's rt_st_* reader (format from the dtypes), copied to the GPU and run
through the C ABI; outputs against the oracle on the original arrays."""
import numpy as np
import pytest

import oracle
from int8_dequant_gemm_b200 import workloads as wl

torch = pytest.importorskip("torch")
st = pytest.importorskip("safetensors.torch")

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def rtq_lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from int8_dequant_gemm_b200 import build
    build.build()
    import int8_dequant_gemm_b200 as rtq
    rtq.lib()
    return rtq


def test_checkpoint_to_gemm(rtq_lib, tmp_path):
    M = 80
    W4, W8, W3 = wl.weights(2048, 512, 11), wl.weights(512, 2048, 12), wl.weights(512, 512, 13)
    q4, q8, f8 = oracle.quant_q4_g32(W4), oracle.quant_q8_row(W8), oracle.quant_e4m3(W3)
    p = tmp_path / "block.safetensors"
    st.save_file({"qkvg": torch.from_numpy(q4[0]),
                  "qkvg.q4_scale": torch.from_numpy(q4[1].view(np.float16)),
                  "w2": torch.from_numpy(q8[0]), "w2.q_scale": torch.from_numpy(q8[1]),
                  "wo": torch.from_numpy(f8).view(torch.float8_e4m3fn)}, str(p))
    X512, X2048 = wl.activations(M, 512, 14), wl.activations(M, 2048, 15)
    with rtq_lib.Checkpoint(p) as ck:
        for name, X, ref in (("qkvg", X512, oracle.gemm_q4(X512, *q4)),
                             ("w2", X2048, oracle.gemm_q8(X2048, *q8)),
                             ("wo", X512, oracle.gemm_e4m3(X512, f8))):
            fmt, codes, scales = ck.weight(name)
            Xd, Wd = torch.from_numpy(X).cuda(), torch.from_numpy(codes).cuda()
            if fmt == rtq_lib.FMT_Q4:
                Y = rtq_lib.qgemm_q4(Xd, Wd, torch.from_numpy(scales).cuda())
            elif fmt == rtq_lib.FMT_Q8:
                Y = rtq_lib.qgemm_q8(Xd, Wd, torch.from_numpy(scales).cuda())
            else:
                Y = rtq_lib.gemm_e4m3(Xd, Wd)
            err = np.max(np.abs(Y.cpu().numpy() - ref)) / np.max(np.abs(ref))
            assert err <= 4e-3, (name, err)
    assert rtq_lib.device_status() == rtq_lib.OK
