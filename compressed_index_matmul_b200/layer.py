"""VQLinear: one compressed layer resident on the GPU plus its library handle."""

from __future__ import annotations

import numpy as np

from . import _binding as B


def _dev(a: np.ndarray, device):
    import torch

    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        a = a.view(np.int16)  # same bits; int16 is torch's portable 16-bit container
    return torch.from_numpy(a).to(device)


class VQLinear:
    """Holds the planes, codebooks and scales of one layer in device memory.

    ``arrays`` is a dict with numpy arrays named as in include/vqlinear.h
    (lo, hi4, s2, idx16, idx8, cb1, cb2, cbr, cb8, scales; fp16 as uint16 bits) and the
    layer shape (N, K, fmt, scale_group).  For the residual ladder (VQ_FMT_VQ16_RVQ)
    idx16 holds one plane per 16-bit stage, cbr is [n16 - 1, 65536, 8] and ``mult``
    the float32 multipliers of the residual stages; the stage counts follow from the
    arrays.  An optional ``corr`` dict (row_ptr int32 [N+1], col int32, val fp16 bits)
    is the sparse correction sidecar; the handle is then created with corr = 1 and
    every forward passes it.  ``forward(x)`` calls vq_linear_forward.
    """

    def __init__(self, N, K, fmt, scale_group, act_dtype, max_M, arrays: dict, device="cuda", rht=0):
        import torch

        self.N, self.K, self.fmt, self.scale_group, self.act_dtype, self.max_M = N, K, fmt, scale_group, act_dtype, max_M
        self.device = torch.device(device)
        self.t = {k: _dev(v, self.device) for k, v in arrays.items() if v is not None and k in
                  ("lo", "hi4", "s2", "idx16", "idx8", "cb1", "cb2", "cbr", "cb8", "scales")}
        self.n16, self.n8, self.mult = 0, 0, ()
        cbr = ()
        if fmt == B.VQ_FMT_VQ16_RVQ:
            ng = N * (K // 8)
            self.n16 = int(np.asarray(arrays["idx16"]).size // ng)
            self.n8 = 1 if arrays.get("idx8") is not None else 0
            self.mult = tuple(float(m) for m in np.asarray(arrays["mult"], dtype=np.float32))
            if "cbr" in self.t:
                stride = 65536 * 8 * 2
                cbr = tuple(self.t["cbr"].data_ptr() + i * stride for i in range(self.n16 - 1))
        self.corr = 0
        if arrays.get("corr") is not None:
            c = arrays["corr"]
            self.corr = 1
            self.t["corr_rows"] = _dev(np.asarray(c["row_ptr"], np.int32), self.device)
            if len(c["col"]):
                self.t["corr_cols"] = _dev(np.asarray(c["col"], np.int32), self.device)
                self.t["corr_vals"] = _dev(np.asarray(c["val"], np.uint16), self.device)
        self.planes = B.make_planes(self.t.get("lo"), self.t.get("hi4"), self.t.get("s2"), self.t.get("idx16"),
                                    self.t.get("idx8"), self.t.get("corr_rows"), self.t.get("corr_cols"),
                                    self.t.get("corr_vals"))
        self.codebooks = B.make_codebooks(self.t["cb1"], self.t.get("cb2"), cbr, self.t.get("cb8"))
        with torch.cuda.device(self.device):
            self.handle = B.vq_linear_create(N, K, fmt, scale_group, act_dtype, max_M, rht, self.n16, self.n8,
                                             self.mult, self.corr)

    @property
    def torch_dtype(self):
        import torch

        return torch.bfloat16 if self.act_dtype == B.VQ_BF16 else torch.float16

    def forward(self, x, y=None, stream=None):
        import torch

        M = x.shape[0]
        if y is None:
            y = torch.empty((M, self.N), dtype=self.torch_dtype, device=self.device)
        B.vq_linear_forward(self.handle, x, self.planes, self.codebooks, self.t["scales"], y, M, self.N, self.K,
                            stream)
        return y

    __call__ = forward

    def forward_rotated(self, x, signs, y=None, stream=None):
        """y = rotate(x) . W^T (vq_linear_forward_rotated); `signs` is an int8 tensor of +-1 [K]."""
        import torch

        M = x.shape[0]
        if y is None:
            y = torch.empty((M, self.N), dtype=self.torch_dtype, device=self.device)
        B.vq_linear_forward_rotated(self.handle, x, signs, self.planes, self.codebooks, self.t["scales"], y, M, self.N,
                                    self.K, stream)
        return y

    def set_path(self, path: int):
        B.vq_linear_set_path(self.handle, path)

    def set_sm_budget(self, sms: int):
        """Run the batch-1 table kernel on at most `sms` SMs (0: all of them)."""
        B.vq_linear_set_sm_budget(self.handle, sms)

    def launches(self, M: int) -> int:
        return B.vq_linear_launches(self.handle, M)

    def plan(self, M: int) -> dict:
        """How a forward of M tokens runs (path, launches, ctas, splits)."""
        return B.vq_linear_plan(self.handle, M)

    def close(self):
        if getattr(self, "handle", None):
            B.vq_linear_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
