"""Per-layer GPTQ on one GPU: the calibration flow of the torchao issue "GPTQ
implementation with tensor subclasses" ("Background": collect the activations
that reach a linear, update its weight with GPTQ, continue with the updated
weight) expressed as three library calls.

`LayerQuantizer` owns the device buffers for one layer shape so that repeated
layers of the same shape reuse them.  All arithmetic happens in libgptq.so;
this module only allocates tensors and sequences calls.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

from . import binding as B


@dataclass
class QuantizedLayer:
    packed: torch.Tensor | None   # uint8 [d_out, d_in/2], even column in the low nibble
    codes: torch.Tensor | None    # uint8 [d_out, d_in], original column order
    scales: torch.Tensor          # float32 [d_out, n_groups], groups in processing order
    zeros: torch.Tensor           # float32 [d_out, n_groups]
    g_idx: torch.Tensor           # int32 [d_in]: group of each original column
    perm: torch.Tensor            # int32 [d_in]: processing order
    W_hat: torch.Tensor           # float32 [d_out, d_in]: dequantized weights
    err_sq: torch.Tensor | None   # float32 [d_out]


class LayerQuantizer:
    def __init__(self, d_out: int, d_in: int, bits: int = 4, group_size: int = 128,
                 block_size: int = 128, damp: float = 0.01, act_order: bool = False,
                 device="cuda", keep_codes: bool = True, keep_err: bool = False):
        self.d_out, self.d_in = d_out, d_in
        self.bits, self.group_size, self.block_size = bits, group_size, block_size
        self.damp, self.act_order = damp, act_order
        dev = torch.device(device)
        self.device = dev
        ng = d_in // group_size if group_size > 0 else 1
        self.H = torch.zeros(d_in, d_in, dtype=torch.float32, device=dev)
        self.U = torch.empty(d_in, d_in, dtype=torch.float32, device=dev)
        self.perm = torch.empty(d_in, dtype=torch.int32, device=dev)
        self.W = torch.empty(d_out, d_in, dtype=torch.float32, device=dev)
        self.scales = torch.empty(d_out, ng, dtype=torch.float32, device=dev)
        self.zeros = torch.empty(d_out, ng, dtype=torch.float32, device=dev)
        self.packed = (torch.empty(d_out, d_in // 2, dtype=torch.uint8, device=dev)
                       if bits <= 4 and d_in % 2 == 0 else None)
        self.codes = torch.empty(d_out, d_in, dtype=torch.uint8, device=dev) if keep_codes else None
        self.g_idx = torch.empty(d_in, dtype=torch.int32, device=dev)
        self.err_sq = torch.empty(d_out, dtype=torch.float32, device=dev) if keep_err else None
        self.ws = B.workspace(d_out, d_in, block_size, device=dev)
        self.staging = None
        self.n_tokens = 0
        self._status = None      # pinned status word of a prepare(wait=False)
        self._pending = False

    # -- step 1: Hessian ------------------------------------------------------
    def reset(self):
        self.H.zero_()
        self.n_tokens = 0

    def add_batch(self, X: torch.Tensor):
        """X bf16 [n, d_in] on the device."""
        B.gptq_hessian_accumulate(self.H, X)
        self.n_tokens += X.shape[0]

    def add_batch_host(self, X_host: torch.Tensor, chunk_tokens: int = 16384):
        """X bf16 [n, d_in] in pinned host memory, copied in overlapped chunks."""
        need = 2 * chunk_tokens * self.d_in
        if self.staging is None or self.staging.numel() < need:
            self.staging = torch.empty(need, dtype=torch.bfloat16, device=self.device)
        B.gptq_hessian_accumulate_host(self.H, X_host, self.staging, chunk_tokens)
        self.n_tokens += X_host.shape[0]

    def add_batch_f32(self, X: torch.Tensor, chunk_tokens: int = 8192):
        """X float32 [n, d_in] on the device (bf16 hi/lo split through the
        tensor-core Hessian; see gptq_hessian_accumulate_f32)."""
        need = B.gptq_hessian_f32_workspace_bytes(self.d_in, chunk_tokens)
        if need == 0:
            raise ValueError("d_in or chunk_tokens out of range for the fp32 Hessian")
        if getattr(self, "ws_f32", None) is None or self.ws_f32.numel() < need:
            self.ws_f32 = torch.empty(need, dtype=torch.uint8, device=self.device)
        B.gptq_hessian_accumulate_f32(self.H, X, self.ws_f32, chunk_tokens)
        self.n_tokens += X.shape[0]

    # -- steps 2-5 ----------------------------------------------------------------
    def prepare(self, wait: bool = True):
        """Damping, activation order and U.  wait=False enqueues the
        factorisation without synchronising the stream (the host can enqueue
        quantize meanwhile); its status is checked by check(), which the next
        prepare also calls."""
        self.check()
        if wait:
            B.gptq_prepare(self.H, self.damp, self.act_order, self.perm, self.U, self.ws)
            return
        if self._status is None:
            self._status = torch.zeros(1, dtype=torch.int32).pin_memory()
            self._done = torch.cuda.Event()
        B.gptq_prepare_async(self.H, self.damp, self.act_order, self.perm, self.U, self.ws,
                             self._status)
        self._done.record(torch.cuda.current_stream(self.device))
        self._pending = True

    def check(self):
        """Raises GptqError if a prepare(wait=False) failed.  Waits only for
        that factorisation (an event after it), not for later work."""
        if not self._pending:
            return
        self._done.synchronize()
        self._pending = False
        st = int(self._status[0])
        if st != 0:
            raise B.GptqError("gptq_prepare_async", st)

    def quantize(self, W: torch.Tensor) -> QuantizedLayer:
        """W [d_out, d_in] bf16 or float32 on the device (not modified)."""
        if W.dtype == torch.bfloat16:
            B.gptq_bf16_to_f32(self.W, W)
        else:
            self.W.copy_(W)
        B.gptq_quantize(self.W, self.U, self.perm if self.act_order else None, self.bits,
                        self.group_size, self.block_size, self.scales, self.zeros, self.ws,
                        codes=self.codes, packed_int4=self.packed, g_idx=self.g_idx,
                        err_sq=self.err_sq)
        return QuantizedLayer(self.packed, self.codes, self.scales, self.zeros, self.g_idx,
                              self.perm, self.W, self.err_sq)

    def quantize_q4k(self, W: torch.Tensor) -> dict:
        """GPTQ onto the two-level Q4_K grid (d_in a multiple of 256; the
        layer's bits / group_size / block_size do not apply).  Returns device
        tensors: codes, packed, g_idx, sc6, m6 (per 32-column block), dsup, dmin
        (per 256-column super-block), scales, offsets (the blocks' d sc and
        dmin m) and W_hat; blocks in processing order."""
        if self.d_in % 256 != 0:
            raise ValueError("the Q4_K grid needs d_in to be a multiple of 256")
        if W.dtype == torch.bfloat16:
            B.gptq_bf16_to_f32(self.W, W)
        else:
            self.W.copy_(W)
        nb, ns = self.d_in // 32, self.d_in // 256
        dev = self.device
        out = {"sc6": torch.empty(self.d_out, nb, dtype=torch.uint8, device=dev),
               "m6": torch.empty(self.d_out, nb, dtype=torch.uint8, device=dev),
               "dsup": torch.empty(self.d_out, ns, dtype=torch.float32, device=dev),
               "dmin": torch.empty(self.d_out, ns, dtype=torch.float32, device=dev),
               "scales": torch.empty(self.d_out, nb, dtype=torch.float32, device=dev),
               "offsets": torch.empty(self.d_out, nb, dtype=torch.float32, device=dev)}
        codes = torch.empty(self.d_out, self.d_in, dtype=torch.uint8, device=dev)
        packed = torch.empty(self.d_out, self.d_in // 2, dtype=torch.uint8, device=dev)
        g_idx = torch.empty(self.d_in, dtype=torch.int32, device=dev)
        B.gptq_quantize_q4k(self.W, self.U, self.perm if self.act_order else None, out, self.ws,
                            codes=codes, packed_int4=packed, g_idx=g_idx)
        out.update(codes=codes, packed=packed, g_idx=g_idx, W_hat=self.W)
        return out

    def quantize_timed(self, W: torch.Tensor):
        """As quantize, enqueued directly (the production launch sequence)
        with the kernels recording their spans; returns (column-loop ms,
        lazy-batch product ms, other ms)."""
        if W.dtype == torch.bfloat16:
            B.gptq_bf16_to_f32(self.W, W)
        else:
            self.W.copy_(W)
        return B.gptq_quantize_timed(self.W, self.U, self.perm if self.act_order else None, self.bits,
                                     self.group_size, self.block_size, self.scales, self.zeros, self.ws,
                                     codes=self.codes, packed_int4=self.packed, g_idx=self.g_idx,
                                     err_sq=self.err_sq)

    def run(self, W: torch.Tensor) -> QuantizedLayer:
        """prepare + quantize.  The column loop is enqueued before the host
        waits for the factorisation's status, so the GPU goes from one to the
        other without a host round trip in between."""
        self.prepare(wait=False)
        out = self.quantize(W)
        self.check()
        return out
