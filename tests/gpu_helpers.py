"""Shared helpers for the GPU tests: device copies of a case, layer params, error metrics."""
import numpy as np
import torch

import pair_representation_b200 as tm

DT = {"bf16": torch.bfloat16, "f32": torch.float32}
FIELDS = ("ln_in_w", "ln_in_b", "w_a", "w_ag", "w_b", "w_bg", "b_a", "b_ag", "b_b", "b_bg",
          "w_g", "b_g", "ln_out_w", "ln_out_b", "w_o", "b_o")


def rel_l2(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.linalg.norm(ref)
    return np.linalg.norm(got - ref) / (den if den > 0 else 1.0)


def max_abs(got, ref):
    return float(np.abs(np.asarray(got, np.float64) - np.asarray(ref, np.float64)).max())


class DeviceCase:
    """A case's arrays on cuda:0 in the given dtype, plus params and a workspace."""

    def __init__(self, case: dict, dtype: str, eps: float = 1e-5, with_mask: bool = True):
        self.dtype = dtype
        tdt = DT[dtype]
        dev = torch.device("cuda", 0)
        self.N = case["z"].shape[0]
        self.z = torch.from_numpy(np.ascontiguousarray(case["z"])).to(dev).to(tdt).contiguous()
        m = case.get("mask") if with_mask else None
        self.mask = None if m is None else torch.from_numpy(np.ascontiguousarray(m)).to(dev).to(tdt).contiguous()
        self.t = {}
        for f in FIELDS:
            v = case.get(f)
            if v is not None:
                self.t[f] = torch.from_numpy(np.ascontiguousarray(v)).to(dev).to(tdt).contiguous()
        code = tm.DTYPE_BF16 if dtype == "bf16" else tm.DTYPE_F32
        self.ws = torch.zeros(tm.trimul_workspace_size_dtype(self.N, 128, 128, code), dtype=torch.uint8, device=dev)
        p = tm.TrimulParams()
        p.N, p.c_z, p.c_h, p.dtype, p.ln_eps = self.N, 128, 128, code, eps
        for f in FIELDS:
            setattr(p, f, self.t[f].data_ptr() if f in self.t else None)
        p.workspace = self.ws.data_ptr()
        p.workspace_bytes = self.ws.numel()
        self.p = p
        self.out = torch.empty_like(self.z)

    def forward(self, direction):
        tm.trimul_forward(self.z, self.mask, self.p, direction, self.out)
        torch.cuda.synchronize()
        rc, detail = tm.trimul_device_status(self.p)
        assert rc == 0, (rc, detail)
        return self.out.float().cpu().numpy()

    def views(self):
        """Workspace sections a, b, x as [128][N][ld] tensors (views, not copies)."""
        a, b, x, ld = tm.trimul_workspace_views(self.p)
        es = 2 if self.dtype == "bf16" else 4
        base = self.ws.data_ptr()
        out = []
        for addr in (a, b, x):
            off = addr - base
            n = 128 * self.N * ld * es
            out.append(self.ws[off:off + n].view(DT[self.dtype]).view(128, self.N, ld))
        return out

    @staticmethod
    def to_cell_major(t, N):
        """[128][N][ld] device tensor -> [N][N][128] float64 numpy."""
        return t[:, :, :N].float().cpu().numpy().transpose(1, 2, 0).astype(np.float64)


def as_bf16(x: np.ndarray) -> np.ndarray:
    """Round float64/float32 values to bf16 (RNE) and return float32 storage."""
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16).float().numpy()
