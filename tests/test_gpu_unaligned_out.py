"""H at a 16-byte but not 32-byte boundary (the C ABI asks for 16).

The long-chunk output kernel then stores H rows in 16-byte pieces instead of
whole 32-byte sectors, and the wide kernel's tensor map starts there.  The
same kernels compute the same values, so the result must equal the aligned
call bit for bit, and nothing may be written outside H (guard elements on
both sides stay zero)."""
import pytest
import torch

from mlstm_chunkwise_b200 import api
from mlstm_chunkwise_b200.inputs import WORKLOADS, make_inputs, scaled

pytestmark = pytest.mark.gpu

CASES = {
    # long chunks, value tiles of 256 columns: one O buffer, epilogue staged in TMEM
    "long_dv512": ("sigmoid_long", dict(B=1, NH=2, T=1536)),
    # long chunks, value tiles of 128 columns: two O buffers, direct stores
    "long_dv128": ("mid", dict(B=1, NH=2, T=1024, chunk_size=512)),
    # chunks of 256: the wide kernel (TMA stores of H)
    "wide_7b": ("xlstm7b", dict(B=1, NH=2, T=1024)),
}


@pytest.mark.parametrize("case", list(CASES))
def test_h_at_a_16_byte_boundary(case):
    base, kw = CASES[case]
    w = scaled(WORKLOADS[base], **kw)
    x = {k: (v.cuda() if v is not None else None) for k, v in make_inputs(w).items()}
    args = (x["Q"], x["K"], x["V"], x["i_pre"], x["f_pre"], x["C0"], x["n0"], x["m0"])
    H_ref, _ = api.mlstm_fw(*args, chunk_size=w.chunk_size, gate_mode=w.gate_mode, algo="tc")
    n = H_ref.numel()
    buf = torch.zeros(n + 16, dtype=H_ref.dtype, device="cuda")
    H = buf[8:8 + n].view(H_ref.shape)  # 8 bf16 = 16 bytes past a 256-byte aligned base
    assert H.data_ptr() % 32 == 16
    api.mlstm_fw(*args, chunk_size=w.chunk_size, gate_mode=w.gate_mode, algo="tc", out={"H": H})
    torch.cuda.synchronize()
    assert torch.equal(H, H_ref)
    assert torch.count_nonzero(buf[:8]) == 0 and torch.count_nonzero(buf[8 + n:]) == 0
