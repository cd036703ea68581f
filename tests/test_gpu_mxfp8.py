"""GPU parity of the MXFP8 contraction (trimul_forward_mxfp8 / trimul_contract_mxfp8).

Reference: oracle/mx.py, the OCP MX v1.0 reading (E4M3 elements in blocks of 32
along the contracted index, E8M0 scale 2^(floor(log2 amax) - 8), round to
nearest even, saturation at 448), pinned on the CPU by tests/test_oracle_mx_pins.py.

Bars:
  * quantizer: bit-exact. Both sides quantize the same bf16 values; amax, the
    scale exponent and the division by a power of two are exact in fp32, and the
    E4M3 rounding is the format's, so every element and every scale byte must
    agree.
  * contraction stage: rel-L2 <= 1e-2 and max-abs <= 4 * 2^-9 * max|ref| (the
    bf16 stage bars). The GPU multiplies the same E4M3 elements and scales
    exactly (8-bit significands), accumulates in fp32 and rounds x to bf16 once.
  * fused prologue (trimul_forward_mxfp8 quantizes inside the prologue): codes
    and scales bit-exact against the oracle's quantization of the bf16 a, b that
    the plain prologue stores for the same inputs.
  * whole layer: the oracle contracts, in MXFP8, the very bf16 a and b the GPU's
    prologue computes (the plain prologue's, read back from the workspace), so both sides take the same
    quantization decisions, then finishes the layer; bars rel-L2 <= 1.5e-2,
    max-abs <= 5e-2 (the bf16 layer bars). (The oracle's own a, b rounded to bf16
    differ from the GPU's by one bf16 ulp in some elements, which flips E4M3
    rounding or a block's scale where a value sits on a boundary: that noise is
    about the size of the bf16 bar itself, so it is not the reference.) Against
    the unquantised float64 layer the error is the format's own: E4M3 keeps 3
    mantissa bits (relative spacing 2^-3, RMS rounding error 2^-3 / sqrt(12) =
    3.6 % per element, about 5 % per product), so x and hence out carry a few
    per cent; the bar there is rel-L2 <= 0.1.
"""
import numpy as np
import pytest
import torch

import oracle
import pair_inputs as pi
import pair_representation_b200 as tm
from gpu_helpers import DeviceCase, as_bf16, max_abs, rel_l2
from oracle.mx import mx_contract, mx_contract_grid, mx_quantize_blocks

pytestmark = pytest.mark.gpu

DIRS = {"outgoing": tm.OUTGOING, "incoming": tm.INCOMING}


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from pair_representation_b200 import build
    build.build()
    tm.lib()


class MxCase(DeviceCase):
    """A DeviceCase whose workspace is sized for the MXFP8 path."""

    def __init__(self, case, **kw):
        super().__init__(case, "bf16", **kw)
        need = tm.trimul_workspace_size_mxfp8(self.N, 128, 128)
        self.ws = torch.zeros(need, dtype=torch.uint8, device=self.z.device)
        self.p.workspace = self.ws.data_ptr()
        self.p.workspace_bytes = need

    def mx_views(self):
        aq, bq, sa, sb, ldq = tm.trimul_mxfp8_views(self.p)
        base = self.ws.data_ptr()
        n = 128 * self.N * ldq
        qa = self.ws[aq - base:aq - base + n].view(128, self.N, ldq)
        qb = self.ws[bq - base:bq - base + n].view(128, self.N, ldq)
        return qa, qb, sa - base, sb - base, ldq


def _operands(N, seed, wide=True):
    """Random bf16 a, b ([N][N][128], cell-major). With `wide`, each value gets a
    random binade in [-12, 12] and some whole rows are zero, so blocks span many
    scales, subnormal E4M3 codes and all-zero blocks."""
    rng = np.random.default_rng([seed, 9])
    out = []
    for _ in range(2):
        v = rng.standard_normal((N, N, 128))
        if wide:
            v *= np.exp2(rng.integers(-12, 13, size=(N, 1, 128)))
            v[rng.uniform(size=N) < 0.05] = 0.0
        out.append(as_bf16(v))
    return out


def _scale_offset(c, r, kb, rows_per_tile, row_tiles, kchunks, chunks_per_tile):
    """Byte offset of the scale of (channel c, operand row r, K block kb), restated
    from the layout the header documents."""
    rt, nl = divmod(r, rows_per_tile)
    chunk = ((c * row_tiles + rt) * kchunks + (kb >> 2)) * chunks_per_tile + (nl >> 7)
    return chunk * 512 + (nl & 31) * 16 + ((nl & 127) >> 5) * 4 + (kb & 3)


def _load(dc, a, b):
    va, vb, vx = dc.views()
    N = dc.N
    va[:, :, :N] = torch.from_numpy(a.transpose(2, 0, 1).copy()).to(va.device).to(torch.bfloat16)
    vb[:, :, :N] = torch.from_numpy(b.transpose(2, 0, 1).copy()).to(vb.device).to(torch.bfloat16)
    vx.fill_(float("nan"))
    return vx


def _assert_codes_match(dc, a, b, direction):
    """The E4M3 codes and scale bytes in dc's MX sections equal the oracle's
    quantization of the bf16 a, b (cell-major [N][N][128]) along the contracted index."""
    N = dc.N
    qa, qb, sa, sb, ldq = dc.mx_views()
    ws = dc.ws.cpu().numpy()
    kc, ti, tj = (N + 127) // 128, (N + 255) // 256, (N + 191) // 192
    axis = 0 if direction == "incoming" else 1  # the contracted index of a and b
    for q, v, soff, rpt, rtiles, cpt in ((qa, a, sa, 128, 2 * ti, 1), (qb, b, sb, 192, tj, 2)):
        P, e, _ = mx_quantize_blocks(v, axis)
        # P, e in operand order: [c][m][k] and [c][m][kb]
        if axis == 1:
            P_op, e_op = P.transpose(2, 0, 1), e.transpose(2, 0, 1)
        else:
            P_op, e_op = P.transpose(2, 1, 0), e.transpose(2, 1, 0)
        got = q[:, :, :N].contiguous().cpu().view(torch.float8_e4m3fn).double().numpy()
        assert np.array_equal(got, P_op), "E4M3 elements differ"
        nb = e_op.shape[2]
        c_i, r_i, k_i = np.meshgrid(np.arange(128), np.arange(N), np.arange(nb), indexing="ij")
        off = _scale_offset(c_i, r_i, k_i, rpt, rtiles, kc, cpt)
        got_e = ws[soff + off].astype(np.int64) - 127
        assert np.array_equal(got_e, e_op.astype(np.int64)), "scale exponents differ"


@pytest.mark.parametrize("N", [33, 200, 385])
@pytest.mark.parametrize("direction", ["outgoing", "incoming"])
def test_mx_quantizer_bit_exact(N, direction):
    a, b = _operands(N, N)
    dc = MxCase(pi.random_case(N, 1, bf16=True, mask="ones"))
    _load(dc, a, b)
    tm.trimul_contract_mxfp8(dc.p, DIRS[direction])
    torch.cuda.synchronize()
    assert tm.trimul_device_status(dc.p)[0] == 0
    _assert_codes_match(dc, a, b, direction)


@pytest.mark.parametrize("N", [33, 200, 385])
@pytest.mark.parametrize("direction", ["outgoing", "incoming"])
@pytest.mark.parametrize("mask", ["random", None])
def test_mx_fused_prologue_bit_exact(N, direction, mask):
    """trimul_forward_mxfp8 quantizes inside the prologue (outgoing on row tiles,
    incoming on 32 x 4 column tiles). Its codes and scales must equal the oracle's
    quantization of the bf16 a, b the plain prologue stores for the same inputs (the
    fused kernel rounds to the same bf16 values before quantizing). Ragged N: partial
    blocks, partial column groups and partial 128-wide K chunks."""
    case = pi.random_case(N, 40 + N, bf16=True, affine=True, mask=mask or "ones")
    dc = MxCase(case, with_mask=mask is not None)
    tm.trimul_prologue(dc.z, dc.mask, dc.p)
    torch.cuda.synchronize()
    a, b = _gpu_ab(dc)
    tm.trimul_forward_mxfp8(dc.z, dc.mask, dc.p, DIRS[direction], dc.out)
    torch.cuda.synchronize()
    assert tm.trimul_device_status(dc.p)[0] == 0
    _assert_codes_match(dc, a, b, direction)


@pytest.mark.parametrize("N", [64, 129, 191, 192, 193, 256, 385, 513, 768])
@pytest.mark.parametrize("direction", ["outgoing", "incoming"])
def test_mx_contraction_stage(N, direction):
    """x from the same bf16 a, b on both sides, against the exact float64 product of
    the oracle's MXFP8 operands: every cell up to N = 385, the sampled grid (every
    192- and 256-wide tile edge, the ragged tail) above."""
    a, b = _operands(N, 1000 + N, wide=False)
    dc = MxCase(pi.random_case(N, 1, bf16=True, mask="ones"))
    vx = _load(dc, a, b)
    tm.trimul_contract_mxfp8(dc.p, DIRS[direction])
    torch.cuda.synchronize()
    assert tm.trimul_device_status(dc.p)[0] == 0
    got = DeviceCase.to_cell_major(vx, N)
    if N <= 385:
        ref = mx_contract(a, b, direction)
    else:
        I = np.unique(np.concatenate([pi.sample_grid(N, N, n_random=8),
                                      [t + d for t in range(192, N, 192) for d in (-1, 0)]])).astype(np.int32)
        ref = mx_contract_grid(a, b, direction, I)
        got = got[np.ix_(I, I)]
    assert np.isfinite(got).all()
    assert rel_l2(got, ref) <= 1e-2
    assert max_abs(got, ref) <= 4 * 2 ** -9 * np.abs(ref).max()


def _gpu_ab(dc):
    """The bf16 a and b the prologue left in the workspace, cell-major float64."""
    va, vb, _ = dc.views()
    return DeviceCase.to_cell_major(va, dc.N), DeviceCase.to_cell_major(vb, dc.N)


def _prologue_ab(dc):
    """The bf16 a and b of the plain prologue on dc's inputs: the values the fused
    MXFP8 prologue rounds to before it quantizes (it stores no bf16 copy)."""
    tm.trimul_prologue(dc.z, dc.mask, dc.p)
    torch.cuda.synchronize()
    return _gpu_ab(dc)


@pytest.mark.parametrize("N,seed", [(100, 11), (300, 12)])
@pytest.mark.parametrize("direction", ["outgoing", "incoming"])
def test_mx_layer(N, seed, direction):
    case = pi.random_case(N, seed, bf16=True, affine=True, mask="random")
    dc = MxCase(case)
    a, b = _prologue_ab(dc)
    tm.trimul_forward_mxfp8(dc.z, dc.mask, dc.p, DIRS[direction], dc.out)
    torch.cuda.synchronize()
    assert tm.trimul_device_status(dc.p)[0] == 0
    got = dc.out.double().cpu().numpy()
    ref = oracle.finish(case, mx_contract(a, b, direction))
    assert rel_l2(got, ref) <= 1.5e-2 and max_abs(got, ref) <= 5e-2
    # The prologue's a, b themselves against the oracle (the bf16 stage bar).
    pa, pb = oracle.project(case)
    assert rel_l2(a, pa) <= 1e-2 and rel_l2(b, pb) <= 1e-2
    exact = oracle.trimul(case, direction)
    assert rel_l2(got, exact) <= 0.1


def test_mx_workload3_sampled():
    """The N = 768 crop in both directions: the MXFP8 layer against the oracle MXFP8
    layer on a sampled grid of cells (the oracle contracts only the sampled rows)."""
    w = pi.WORKLOADS[3]
    case = pi.make_workload(w)
    dc = MxCase(case)
    I = pi.sample_grid(w.N, w.seed, n_random=8)
    a, b = _prologue_ab(dc)
    for direction in w.directions:
        tm.trimul_forward_mxfp8(dc.z, dc.mask, dc.p, DIRS[direction], dc.out)
        torch.cuda.synchronize()
        assert tm.trimul_device_status(dc.p)[0] == 0
        got = dc.out.double().cpu().numpy()[np.ix_(I, I)]
        x = mx_contract_grid(a, b, direction, I)
        sub = {k: v for k, v in case.items() if k not in ("z", "mask", "m")}
        sub["z"] = case["z"][np.ix_(I, I)]
        ref = oracle.finish(sub, x)
        assert rel_l2(got, ref) <= 1.5e-2 and max_abs(got, ref) <= 5e-2, direction


def test_mx_rejects_small_workspace_and_fp32():
    case = pi.random_case(64, 3, bf16=True, mask="ones")
    dc = DeviceCase(case, "bf16")  # bf16-sized workspace: too small for the MXFP8 sections
    rc = tm.trimul_forward_mxfp8(dc.z, dc.mask, dc.p, tm.OUTGOING, dc.out, check=False)
    assert rc == tm.ERR["TRIMUL_ERR_WORKSPACE"]
    f = DeviceCase(pi.random_case(64, 3, mask="ones"), "f32")
    rc = tm.trimul_forward_mxfp8(f.z, f.mask, f.p, tm.OUTGOING, f.out, check=False)
    assert rc == tm.ERR["TRIMUL_ERR_UNSUPPORTED"]


@pytest.mark.parametrize("direction", ["outgoing", "incoming"])
def test_mx_stage_calls_compose(direction):
    """trimul_prologue_mxfp8, trimul_mma_mxfp8 and trimul_epilogue on one stream give
    bit for bit what trimul_forward_mxfp8 gives."""
    N = 257
    case = pi.random_case(N, 77, bf16=True, affine=True, mask="random")
    dc = MxCase(case)
    tm.trimul_forward_mxfp8(dc.z, dc.mask, dc.p, DIRS[direction], dc.out)
    torch.cuda.synchronize()
    whole = dc.out.clone()
    dc.out.fill_(float("nan"))
    tm.trimul_prologue_mxfp8(dc.z, dc.mask, dc.p, DIRS[direction])
    tm.trimul_mma_mxfp8(dc.p)
    tm.trimul_epilogue(dc.z, dc.p, dc.out)
    torch.cuda.synchronize()
    assert tm.trimul_device_status(dc.p)[0] == 0
    assert torch.equal(whole, dc.out)
