"""Device-resident decode problems: upload a workload, own the buffers, call
the C ABI.  Torch is used for device memory and streams only.
"""

from __future__ import annotations

import numpy as np

from . import kvattn as K


def bf16_tensor(bits: np.ndarray, device):
    """uint16 bf16 bit patterns -> torch.bfloat16 tensor on ``device``."""
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)


class DeviceProblem:
    """One decode batch resident in HBM plus its out / lse / workspace buffers."""

    def __init__(self, inputs: dict, device="cuda", num_splits: int = 0, max_seq_len: int | None = None):
        import torch
        s = inputs["shape"]
        self.shape = s
        self.device = torch.device(device)
        self.variant = K.VARIANTS[s.variant]
        self.q_nope = bf16_tensor(inputs["q_nope"], self.device)
        self.q_rope = None if inputs["q_rope"] is None else bf16_tensor(inputs["q_rope"], self.device)
        if getattr(s, "cache_dtype", "bf16") == "fp8":
            self.kv = torch.from_numpy(np.ascontiguousarray(inputs["kv"], dtype=np.uint8)).to(self.device)
        else:
            self.kv = bf16_tensor(inputs["kv"], self.device)
        bt = inputs["block_table"]
        self.block_table = None if bt is None else torch.from_numpy(bt).to(self.device)
        self.seq_lens = torch.from_numpy(np.asarray(inputs["seq_lens"], np.int32)).to(self.device)
        if max_seq_len is None:
            max_seq_len = int(np.max(inputs["seq_lens"])) if len(inputs["seq_lens"]) else 0
        self.max_seq_len = max_seq_len
        self.sm_scale = float(inputs["sm_scale"])
        self.num_pages = int(inputs["num_pages"])
        self.max_pages_per_seq = int(inputs["max_pages_per_seq"])
        self.params = K.params_for(s, self.max_pages_per_seq, self.num_pages, max_seq_len, num_splits)
        self.plan = K.kvattn_get_plan(self.variant, self.params)
        self.workspace = torch.empty(int(self.plan.workspace_bytes), dtype=torch.uint8, device=self.device)
        st = K.kvattn_workspace_init(self.workspace.data_ptr(), self.workspace.numel(),
                                     torch.cuda.current_stream(self.device).cuda_stream)
        if st:
            raise K.KvattnError(st, "kvattn_workspace_init")
        out_dtype = torch.float32 if s.out_dtype == "fp32" else torch.bfloat16
        self.out = torch.empty(s.out_shape(), dtype=out_dtype, device=self.device)
        self.lse = torch.empty(s.lse_shape(), dtype=torch.float32, device=self.device)

    def run(self, stream=None, out=None, lse=None, q_nope=None, q_rope=None, seq_lens=None,
            block_table=None, events=None):
        """Enqueue one decode call (optionally on other q / out buffers)."""
        K.decode_tensors(self.variant, self.params,
                         self.q_nope if q_nope is None else q_nope,
                         self.q_rope if q_rope is None else q_rope,
                         self.kv,
                         self.block_table if block_table is None else block_table,
                         self.seq_lens if seq_lens is None else seq_lens,
                         self.sm_scale,
                         self.out if out is None else out,
                         self.lse if lse is None else lse,
                         self.workspace, stream, events)

    def append_kv(self, new_kv, pos, rope_base, device_error=None, stream=None):
        """Write new token rows into this problem's cache (kvattn_append_kv)."""
        import torch
        st = K.kvattn_append_kv(self.variant, self.params, new_kv.data_ptr(), pos.data_ptr(),
                                None if self.block_table is None else self.block_table.data_ptr(),
                                self.kv.data_ptr(), rope_base,
                                None if device_error is None else device_error.data_ptr(),
                                torch.cuda.current_stream(self.device).cuda_stream if stream is None else stream)
        if st:
            raise K.KvattnError(st, "kvattn_append_kv")

    def plan_kernel_name(self) -> str:
        return K.KERNEL_NAMES.get(int(self.plan.kernel), str(self.plan.kernel))

    def device_error(self) -> int:
        import torch
        return K.kvattn_get_device_error(self.workspace.data_ptr(),
                                         torch.cuda.current_stream(self.device).cuda_stream)

    def clear_device_error(self):
        import torch
        K.kvattn_workspace_init(self.workspace.data_ptr(), self.workspace.numel(),
                                torch.cuda.current_stream(self.device).cuda_stream)

    def results(self):
        """(out, lse) as float64 numpy arrays."""
        return (self.out.float().cpu().numpy().astype(np.float64),
                self.lse.cpu().numpy().astype(np.float64))
