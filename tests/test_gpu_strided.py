"""Row-strided sequence tensors: esa_scan_fwd_ld and esa_scan_bwd_ld.

a, v, q are the column blocks of one ``[B, T, 3 C + pad]`` buffer, the way a
single projection GEMM lays them out, and da, dv, dq are written into the
column blocks of another such buffer.  The results must be bitwise those of
the contiguous calls on copies of the same values (the arithmetic is the
same, only the addresses differ), the padding columns of the gradient buffer
must be left as they were, and the oracle must agree.  Every I/O dtype and
tile width, ragged lengths, partial channel tiles.
"""
import pytest
import torch

from gated_linear_recurrence_b200 import esa, inputs
from tests._parity import DT, TOL, compare, oracle_fwd_bwd

pytestmark = pytest.mark.gpu

F8 = torch.float8_e4m3fn
CASES = [
    # B, T, H, D, mode, dtype, pad of the input rows, pad of the gradient rows (elements)
    (2, 1000, 4, 32, 1, "f16", 0, 0),
    (2, 333, 5, 16, 0, "bf16", 8, 24),     # C = 80: two channel tiles, the second partial
    (1, 300, 2, 128, 1, "f32", 4, 12),
    (2, 257, 1, 256, 0, "f16", 16, 8),
    (3, 129, 16, 8, 1, "bf16", 0, 8),      # D = 8: one lane per head
    (2, 500, 4, 32, 0, "e4m3", 16, 8),     # 1-byte inputs, fp16 gradients
]
SENTINEL = 1000.0   # exact in every output type


def _ids(c):
    return f"B{c[0]}T{c[1]}H{c[2]}D{c[3]}m{c[4]}{c[5]}pad{c[6]}-{c[7]}"


def _blocks(buf, B, T, H, D):
    C = H * D
    return [buf[..., i * C:(i + 1) * C].view(B, T, H, D) for i in range(3)]


@pytest.mark.parametrize("case", CASES, ids=[_ids(c) for c in CASES])
def test_strided_scans_equal_contiguous_scans(cuda_device, case):
    B, T, H, D, mode, dt, pad_in, pad_g = case
    C = H * D
    io = F8 if dt == "e4m3" else DT[dt]
    x = inputs.make_scan_inputs(B, T, H, D, "f32" if dt == "e4m3" else dt, 1.5, 500 + T)
    xd = {k: x[k].to(io).to(cuda_device) for k in ("a", "v", "q", "dy")}
    E0 = inputs.make_state(B, H, D, seed=501, scale=0.5).to(cuda_device)
    dEf = inputs.make_state(B, H, D, seed=502).to(cuda_device)

    X = torch.zeros(B, T, 3 * C + pad_in, dtype=io, device=cuda_device)
    sa, sv, sq = _blocks(X, B, T, H, D)
    for dst, k in ((sa, "a"), (sv, "v"), (sq, "q")):
        dst.copy_(xd[k])
    assert esa.row_stride(sa) == 3 * C + pad_in

    y_s, Ef_s, ws_s = esa.esa_scan_fwd(sa, sv, sq, mode=mode, E_init=E0)
    y_c, Ef_c, ws_c = esa.esa_scan_fwd(xd["a"], xd["v"], xd["q"], mode=mode, E_init=E0)
    odt = esa.out_dtype(io)
    G = torch.full((B, T, 3 * C + pad_g), SENTINEL, dtype=odt, device=cuda_device)
    ga, gv, gq = _blocks(G, B, T, H, D)
    _, _, _, dE0_s = esa.esa_scan_bwd(sa, sv, sq, xd["dy"], ws_s, mode=mode, E_init=E0, dE_final=dEf,
                                      da=ga, dv=gv, dq=gq)
    da_c, dv_c, dq_c, dE0_c = esa.esa_scan_bwd(xd["a"], xd["v"], xd["q"], xd["dy"], ws_c, mode=mode, E_init=E0,
                                               dE_final=dEf)
    esa.esa_check(ws_s)
    esa.esa_check(ws_c)
    for name, s_, c_ in (("y", y_s, y_c), ("E_final", Ef_s, Ef_c), ("da", ga, da_c), ("dv", gv, dv_c),
                         ("dq", gq, dq_c), ("dE_init", dE0_s, dE0_c)):
        assert torch.equal(s_, c_), f"{name}: strided and contiguous results differ"
    if pad_g:
        assert bool((G[..., 3 * C:] == SENTINEL).all()), "a padding column of the gradient rows was written"

    widened = {k: t.float() for k, t in xd.items()}    # the values the kernels read, exactly
    ref = oracle_fwd_bwd(widened, mode, E_init=E0, dE_final=dEf)
    gpu = {"y": y_s, "E_final": Ef_s, "da": ga, "dv": gv, "dq": gq, "dE_init": dE0_s}
    compare(gpu, ref, TOL[odt if dt == "e4m3" else DT[dt]], tuple(gpu))


def test_strided_arguments_are_checked(cuda_device):
    B, T, H, D = 2, 64, 4, 32
    C = H * D
    X = torch.zeros(B, T, 3 * C, dtype=torch.float16, device=cuda_device)
    a, v, q = _blocks(X, B, T, H, D)
    other = torch.zeros(B, T, 2 * C, dtype=torch.float16, device=cuda_device)[..., :C].view(B, T, H, D)
    with pytest.raises(ValueError, match="one row stride"):
        esa.esa_scan_fwd(a, v, other)
    with pytest.raises(ValueError, match="channels contiguous"):
        esa.esa_scan_fwd(a, v, torch.zeros(B, T, D, H, dtype=torch.float16, device=cuda_device).transpose(2, 3))
    odd = torch.zeros(B, T, 3 * C + 1, dtype=torch.float16, device=cuda_device)
    oa, ov, oq = (odd[..., i * C:(i + 1) * C].view(B, T, H, D) for i in range(3))
    with pytest.raises(esa.EsaError) as err:   # rows of 385 halves: not whole 16-byte units
        esa.esa_scan_fwd(oa, ov, oq)
    assert err.value.code in (esa.ESA_ERR_ALIGN, esa.ESA_ERR_ARG)
