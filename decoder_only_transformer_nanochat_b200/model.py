"""Convenience wrapper over the C ABI that uses PyTorch only for device memory
and the current CUDA stream.  Every computation is done by the CUDA library."""
from __future__ import annotations

import torch

from . import _binding as B


class Model:
    """One nanochat decoder of the given depth (one dial: width = depth*64,
    heads = width/128) on the current CUDA device."""

    def __init__(self, depth: int, vocab: int = 65536, seq: int = 2048, dtype: str = "bf16",
                 window: int = 0, value_embeds: bool = False, resid_scalars: bool = False):
        """window / value_embeds / resid_scalars: the full reference block's
        options (sliding-window "SSSL" layers, gated value embeddings,
        residual scalars); all off is the baseline decoder."""
        self.dtype_code = B.NC_BF16 if dtype == "bf16" else B.NC_F32
        self.torch_dtype = torch.bfloat16 if dtype == "bf16" else torch.float32
        rc, self.handle = B.nc_init_ex(depth, vocab, seq, self.dtype_code, window, value_embeds,
                                       resid_scalars)
        if rc != B.NC_OK:
            raise B.NcError(rc, "nc_init_ex")
        rc, self.dims = B.nc_get_dims(self.handle)
        if rc != B.NC_OK:
            raise B.NcError(rc, "nc_get_dims")
        rc, n = B.nc_param_count(self.handle)
        if rc != B.NC_OK:
            raise B.NcError(rc, "nc_param_count")
        self.windows = [B.nc_layer_window(self.handle, l)[1] for l in range(depth)]
        self.layout = []
        for i in range(n):
            rc, p = B.nc_param_layout(self.handle, i)
            if rc != B.NC_OK:
                raise B.NcError(rc, "nc_param_layout")
            self.layout.append(p)
        self.n_params = self.dims["n_params"]
        self._ws = None
        self._ws_key = None

    def __del__(self):
        h = getattr(self, "handle", None)
        if h:
            B.nc_destroy(h)
            self.handle = None

    def workspace(self, Bsz: int, T: int) -> torch.Tensor:
        rc, n = B.nc_workspace_bytes(self.handle, Bsz, T)
        if rc != B.NC_OK:
            raise B.NcError(rc, "nc_workspace_bytes")
        if self._ws is None or self._ws.numel() < n:
            self._ws = None
            self._ws = torch.empty(n, dtype=torch.uint8, device="cuda")
        return self._ws

    @staticmethod
    def _stream():
        return torch.cuda.current_stream().cuda_stream

    def fwd_bwd(self, weights: torch.Tensor, tokens: torch.Tensor, targets: torch.Tensor,
                grads: torch.Tensor | None = None, loss: torch.Tensor | None = None,
                token_loss: torch.Tensor | None = None, accumulate: bool = False):
        """Loss and gradients of one step; accumulate=True adds the gradients
        to `grads` instead of writing over them."""
        Bsz, T = tokens.shape
        ws = self.workspace(Bsz, T)
        if grads is None:
            if accumulate:
                raise ValueError("accumulate needs the gradient buffer to add to")
            grads = torch.empty(self.n_params, dtype=torch.float32, device="cuda")
        if loss is None:
            loss = torch.empty(1, dtype=torch.float32, device="cuda")
        rc = B.nc_fwd_bwd_ex(self.handle, weights.data_ptr(), tokens.data_ptr(), targets.data_ptr(),
                             Bsz, T, ws.data_ptr(), ws.numel(), loss.data_ptr(),
                             token_loss.data_ptr() if token_loss is not None else None,
                             grads.data_ptr(), B.NC_ACCUMULATE if accumulate else 0, self._stream())
        if rc != B.NC_OK:
            raise B.NcError(rc, "nc_fwd_bwd_ex")
        return loss, grads

    def grad_buckets(self):
        """[(offset, count)] of the gradient buffer, in the order the backward finishes them."""
        rc, b = B.nc_grad_buckets(self.handle)
        if rc != B.NC_OK:
            raise B.NcError(rc, "nc_grad_bucket")
        return b

    def set_grad_events(self, events) -> None:
        rc = B.nc_set_grad_events(self.handle, events)
        if rc != B.NC_OK:
            raise B.NcError(rc, "nc_set_grad_events")

    def fwd(self, weights: torch.Tensor, tokens: torch.Tensor, logits: torch.Tensor | None = None):
        Bsz, T = tokens.shape
        ws = self.workspace(Bsz, T)
        if logits is None:
            logits = torch.empty(Bsz, T, self.dims["vocab"], dtype=self.torch_dtype, device="cuda")
        rc = B.nc_fwd(self.handle, weights.data_ptr(), tokens.data_ptr(), Bsz, T, ws.data_ptr(),
                      ws.numel(), logits.data_ptr(), self._stream())
        if rc != B.NC_OK:
            raise B.NcError(rc, "nc_fwd")
        return logits

    # ---------------- optimizer ----------------

    def optimizer_state(self, weights: torch.Tensor) -> torch.Tensor:
        """fp32 state (master copy, moments) initialised from the weights."""
        rc, n = B.nc_optim_state_bytes(self.handle)
        if rc != B.NC_OK:
            raise B.NcError(rc, "nc_optim_state_bytes")
        state = torch.empty(n // 4, dtype=torch.float32, device="cuda")
        rc = B.nc_optim_init(self.handle, weights.data_ptr(), state.data_ptr(), self._stream())
        if rc != B.NC_OK:
            raise B.NcError(rc, "nc_optim_init")
        return state

    def optimizer_step(self, weights: torch.Tensor, grads: torch.Tensor, state: torch.Tensor, step: int,
                       opts: dict) -> None:
        """One Muon / AdamW step.  opts: every field of nc_optim_opts (lr_matrix,
        lr_embed, lr_head, lr_scalar, weight_decay, muon_momentum, ns_steps,
        beta1, beta2, eps); the pages give no values, so there are no defaults."""
        rc, n = B.nc_optim_workspace_bytes(self.handle)
        if rc != B.NC_OK:
            raise B.NcError(rc, "nc_optim_workspace_bytes")
        if getattr(self, "_ows", None) is None or self._ows.numel() < n:
            self._ows = torch.empty(n, dtype=torch.uint8, device="cuda")
        rc = B.nc_optim_step(self.handle, weights.data_ptr(), grads.data_ptr(), state.data_ptr(), step, opts,
                             self._ows.data_ptr(), self._ows.numel(), self._stream())
        if rc != B.NC_OK:
            raise B.NcError(rc, "nc_optim_step")

    # ---------------- inference with a KV cache ----------------

    def kv_cache(self, Bsz: int, T_max: int):
        """A zeroed KV cache for Bsz rows of up to T_max positions, and the
        per-row sequence lengths (device int32)."""
        rc, n = B.nc_kv_cache_bytes(self.handle, Bsz, T_max)
        if rc != B.NC_OK:
            raise B.NcError(rc, "nc_kv_cache_bytes")
        return (torch.zeros(n, dtype=torch.uint8, device="cuda"),
                torch.zeros(Bsz, dtype=torch.int32, device="cuda"))

    def prefill(self, weights: torch.Tensor, tokens: torch.Tensor, cache, T_max: int):
        """Forward over the prompts tokens [B, T]; fills the cache; returns the
        softcapped logits of each row's last position [B, vocab]."""
        Bsz, T = tokens.shape
        kv, seqlens = cache
        ws = self.workspace(Bsz, T)
        logits = torch.empty(Bsz, self.dims["vocab"], dtype=self.torch_dtype, device="cuda")
        rc = B.nc_prefill(self.handle, weights.data_ptr(), tokens.data_ptr(), Bsz, T, kv.data_ptr(), T_max,
                          seqlens.data_ptr(), ws.data_ptr(), ws.numel(), logits.data_ptr(), self._stream())
        if rc != B.NC_OK:
            raise B.NcError(rc, "nc_prefill")
        return logits

    def decode(self, weights: torch.Tensor, tokens: torch.Tensor, cache, T_max: int):
        """One token per row (tokens [B]) at each row's next position; returns
        its softcapped logits [B, vocab]."""
        Bsz = tokens.shape[0]
        kv, seqlens = cache
        ws = self.workspace(Bsz, 1)
        logits = torch.empty(Bsz, self.dims["vocab"], dtype=self.torch_dtype, device="cuda")
        rc = B.nc_decode(self.handle, weights.data_ptr(), tokens.data_ptr(), Bsz, kv.data_ptr(), T_max,
                         seqlens.data_ptr(), ws.data_ptr(), ws.numel(), logits.data_ptr(), self._stream())
        if rc != B.NC_OK:
            raise B.NcError(rc, "nc_decode")
        return logits

    def sync_status(self, timeout_ms: int = 60000) -> int:
        return B.nc_sync_status(self.handle, self._stream(), timeout_ms)
