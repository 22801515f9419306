"""Torch-tensor front end of libmfsdp: marshals tensors into the C ABI.

PyTorch provides device memory and streams only.  Every step of the update
runs in the library's kernels; nothing here computes on tensor values.
"""

from __future__ import annotations

from typing import List, Optional, Sequence

import torch

from . import _lib

_DT = {torch.float32: _lib.MFSDP_DTYPE_F32, torch.bfloat16: _lib.MFSDP_DTYPE_BF16}


def _dtype_code(t: torch.Tensor) -> int:
    try:
        return _DT[t.dtype]
    except KeyError:
        raise TypeError(f"unsupported dtype {t.dtype}; libmfsdp takes float32 or bfloat16") from None


def _check_tensor(t: torch.Tensor, name: str) -> None:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous (row-major)")


def _stream_handle(stream: Optional[torch.cuda.Stream]) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return int(s.cuda_stream)


class MuonOwnerStep:
    """The owner's grouped Muon step over a fixed list of matrices.

    ``params``, ``grads``, ``momenta`` are same-shape 2D CUDA tensors per matrix
    (params/grads float32 or bfloat16, momenta float32).  ``update_outs`` may
    hold float32 tensors that receive the update O (tests), or None.
    """

    def __init__(self, params: Sequence[torch.Tensor], grads: Sequence[Optional[torch.Tensor]],
                 momenta: Sequence[torch.Tensor], update_outs: Optional[Sequence[Optional[torch.Tensor]]] = None,
                 lr: float = 0.02, beta: float = 0.95, weight_decay: float = 0.01, eps: float = 1e-7,
                 a: float = 3.4445, b: float = -4.7750, c: float = 2.0315, ns_steps: int = 5,
                 nesterov: bool = True, mode: str = "bf16",
                 grad_parts: Optional[Sequence[Sequence[torch.Tensor]]] = None,
                 param_copies: Optional[Sequence[Sequence[torch.Tensor]]] = None,
                 overlap_groups: int = 0):
        """``grad_parts[i]`` (optional): the ranks' contributions to matrix i's
        gradient, summed in order inside the step (``grads[i]`` may then be
        None); ``param_copies[i]``: tensors that receive the updated parameter.
        Either list turns the call into mfsdp_muon_step_p2p; the tensors may live
        on peer GPUs that this device can access.  ``overlap_groups`` > 0 runs
        mfsdp_muon_step_p2p_overlap instead: the list in that many groups, each
        group's copies on a side stream (the copy engines) while later groups
        compute."""
        if not (len(params) == len(grads) == len(momenta)):
            raise ValueError("params, grads and momenta must have the same length")
        if update_outs is None:
            update_outs = [None] * len(params)
        self.mode = {"bf16": _lib.MFSDP_MODE_BF16, "fp32": _lib.MFSDP_MODE_FP32}[mode]
        self.hp = _lib.muon_hparams(lr, beta, weight_decay, eps, a, b, c, ns_steps, nesterov, self.mode)
        p2p = grad_parts is not None or param_copies is not None
        if p2p:
            grad_parts = grad_parts if grad_parts is not None else [[g] for g in grads]
            param_copies = param_copies if param_copies is not None else [[] for _ in params]
        mats: List[_lib.Matrix] = []
        for i, (w, g, m, o) in enumerate(zip(params, grads, momenta, update_outs)):
            if p2p and g is None:
                g = grad_parts[i][0]
            for t, nm in ((w, "param"), (g, "grad"), (m, "momentum")):
                _check_tensor(t, f"{nm}[{i}]")
            if w.dim() != 2 or w.shape != g.shape or w.shape != m.shape:
                raise ValueError(f"matrix {i}: param, grad and momentum must be 2D of equal shape")
            if p2p:
                for t in list(grad_parts[i]) + list(param_copies[i]):
                    _check_tensor(t, f"segment tensor of matrix {i}")
                    if t.shape != w.shape:
                        raise ValueError(f"matrix {i}: grad parts and param copies must have the param's shape")
                if any(t.dtype != g.dtype for t in grad_parts[i]) or any(t.dtype != w.dtype for t in param_copies[i]):
                    raise TypeError(f"matrix {i}: parts take the grad dtype, copies the param dtype")
            if m.dtype != torch.float32:
                raise TypeError(f"momentum[{i}] must be float32")
            if o is not None:
                _check_tensor(o, f"update_out[{i}]")
                if o.shape != w.shape or o.dtype != torch.float32:
                    raise ValueError(f"update_out[{i}] must be float32 of the param's shape")
            mats.append(_lib.Matrix(w.data_ptr(), g.data_ptr(), m.data_ptr(),
                                    o.data_ptr() if o is not None else None,
                                    w.shape[0], w.shape[1], _dtype_code(w), _dtype_code(g)))
        self._tensors = (list(params), list(grads), list(momenta), list(update_outs), grad_parts, param_copies)
        self.mats = mats
        self._arr = _lib.matrix_array(mats)
        self._segs = None
        self.overlap_groups = int(overlap_groups)
        if self.overlap_groups and not p2p:
            raise ValueError("overlap_groups needs grad_parts or param_copies")
        if p2p:
            self._segs, self._seg_keep = _lib.owner_segments(
                [[t.data_ptr() for t in parts] for parts in grad_parts],
                [[t.data_ptr() for t in copies] for copies in param_copies])
            if self.overlap_groups:
                self.workspace_bytes = _lib.mfsdp_muon_workspace_size_p2p_overlap(mats, self._segs, self.hp,
                                                                                  self.overlap_groups)
            else:
                self.workspace_bytes = _lib.mfsdp_muon_workspace_size_p2p(mats, self._segs, self.hp)
        else:
            self.workspace_bytes = _lib.mfsdp_muon_workspace_size(mats, self.hp)
        dev = params[0].device if len(params) else torch.device("cuda")
        # 256-byte aligned workspace carved from a torch allocation
        self._ws = torch.empty(self.workspace_bytes + 256, dtype=torch.uint8, device=dev)
        base = self._ws.data_ptr()
        self.workspace_ptr = (base + 255) // 256 * 256
        self.launches = _lib.mfsdp_muon_step_launches(mats, self.hp)
        self._copy_stream = torch.cuda.Stream(device=dev) if self.overlap_groups else None

    def step(self, stream: Optional[torch.cuda.Stream] = None) -> None:
        if self._segs is not None and self.overlap_groups:
            _lib.mfsdp_muon_step_p2p_overlap(self.mats, self._segs, self.hp, self.overlap_groups,
                                             self.workspace_ptr, self.workspace_bytes, _stream_handle(stream),
                                             int(self._copy_stream.cuda_stream), arr=self._arr)
        elif self._segs is not None:
            _lib.mfsdp_muon_step_p2p(self.mats, self._segs, self.hp, self.workspace_ptr, self.workspace_bytes,
                                     _stream_handle(stream), arr=self._arr)
        else:
            _lib.mfsdp_muon_step(self.mats, self.hp, self.workspace_ptr, self.workspace_bytes,
                                 _stream_handle(stream), arr=self._arr)

    def capture_graph(self) -> "torch.cuda.CUDAGraph":
        """One step captured into a CUDA graph; ``replay()`` reruns it on the same
        tensors with the same hyper-parameters.  Call ``step()`` once before
        capturing: the workspace's descriptor table is then already on the
        device, and the capture holds only the step's kernel launches."""
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            self.step()
        return g

    def close(self) -> None:
        if getattr(self, "_ws", None) is not None:
            _lib.mfsdp_muon_forget_workspace_range(self.workspace_ptr, max(self.workspace_bytes, 1))
            self._ws = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def adamw_tail(p: torch.Tensor, g: torch.Tensor, m: torch.Tensor, v: torch.Tensor, step: int,
               lr: float = 0.02, beta1: float = 0.9, beta2: float = 0.95, eps: float = 1e-8,
               weight_decay: float = 0.01, stream: Optional[torch.cuda.Stream] = None) -> None:
    """AdamW over a flat packed fp32 tail (all four tensors 1D, same length)."""
    for t, nm in ((p, "p"), (g, "g"), (m, "m"), (v, "v")):
        _check_tensor(t, nm)
        if t.dtype != torch.float32:
            raise TypeError(f"{nm} must be float32")
        if t.numel() != p.numel():
            raise ValueError("tail tensors must have equal length")
    hp = _lib.adamw_hparams(lr, beta1, beta2, eps, weight_decay, step)
    _lib.mfsdp_adamw_tail(p.data_ptr(), g.data_ptr(), m.data_ptr(), v.data_ptr(), p.numel(), hp,
                          _stream_handle(stream))


def device_status(stream: Optional[torch.cuda.Stream] = None) -> int:
    return _lib.mfsdp_get_device_status(_stream_handle(stream))
