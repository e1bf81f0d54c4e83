"""A torch.nn.Module drop-in for nn.Linear with 4-bit weights.

The page "Building a pure-Python INT4 transformer weight quantizer with
block-wise per-channel scaling" lists, among its extensions, a
torch.nn.Module wrapper over the INT4 weights for drop-in replacement, with
the scales persisted alongside the weights; the page "Build a Blockwise INT4
Inference Engine" (step 4) has the layer: y = x @ W_dq^T + bias, then ReLU
(its step 3 fuses the ReLU into the kernel).  Int4Linear holds the packed
codes, the fp16 scales (and, for the affine scheme, the zero points) as
buffers, so state_dict() carries them, and calls the library's fused matmul
with the bias and the optional ReLU in its epilogue.  All arithmetic runs in
the library's CUDA kernels.
"""

from __future__ import annotations

import torch

from . import int4_matmul, quantize_int4, quantize_int4_affine

__all__ = ["Int4Linear"]


class Int4Linear(torch.nn.Module):
    """y = act(x @ dequantize(W)^T + bias) with W [out_features, in_features]
    stored as 4-bit codes.

    scheme: "symmetric" (the drill's scheme: two's-complement codes, scale =
    absmax / 7) or "affine" (unsigned codes with per-group zero points).
    relu: apply ReLU after the bias, fused into the matmul's store.
    out_dtype: dtype of the output (default: the input's dtype); the matmul
    itself produces fp32.
    """

    def __init__(self, in_features: int, out_features: int, *, bias: bool = True,
                 group: int = 128, scheme: str = "symmetric", relu: bool = False,
                 device=None, out_dtype: torch.dtype | None = None):
        super().__init__()
        if scheme not in ("symmetric", "affine"):
            raise ValueError("scheme must be 'symmetric' or 'affine'")
        if in_features < 1 or out_features < 1 or group < 1:
            raise ValueError("in_features, out_features and group must be >= 1")
        self.in_features, self.out_features = int(in_features), int(out_features)
        self.group, self.scheme, self.relu, self.out_dtype = int(group), scheme, bool(relu), out_dtype
        G = -(-self.in_features // self.group)
        dev = torch.device("cuda") if device is None else torch.device(device)
        self.register_buffer("packed", torch.zeros((self.out_features, (self.in_features + 1) // 2),
                                                   dtype=torch.uint8, device=dev))
        self.register_buffer("scales", torch.zeros((self.out_features, G), dtype=torch.float16,
                                                   device=dev))
        if scheme == "affine":
            self.register_buffer("zeros", torch.zeros((self.out_features, G), dtype=torch.uint8,
                                                      device=dev))
        else:
            self.zeros = None
        if bias:
            self.register_buffer("bias", torch.zeros(self.out_features, dtype=torch.float32,
                                                     device=dev))
        else:
            self.bias = None

    @torch.no_grad()
    def load_weight(self, weight: torch.Tensor, bias: torch.Tensor | None = None) -> "Int4Linear":
        """Quantize `weight` [out_features, in_features] (fp32/bf16/fp16, on the
        GPU) into the module's buffers; copy `bias` if given."""
        if tuple(weight.shape) != (self.out_features, self.in_features):
            raise ValueError("weight must be [out_features, in_features]")
        w = weight.detach().to(self.packed.device).contiguous()
        if self.scheme == "affine":
            quantize_int4_affine_into(w, self.group, self.packed, self.scales, self.zeros)
        else:
            quantize_int4(w, self.group, packed=self.packed, scales=self.scales)
        if bias is not None:
            if self.bias is None:
                raise ValueError("this layer has no bias")
            self.bias.copy_(bias.detach().to(torch.float32))
        return self

    @classmethod
    def from_linear(cls, linear: torch.nn.Linear, *, group: int = 128, scheme: str = "symmetric",
                    relu: bool = False, device=None, out_dtype=None) -> "Int4Linear":
        """An Int4Linear holding the quantized weight and the bias of `linear`."""
        dev = device if device is not None else (linear.weight.device if linear.weight.is_cuda
                                                 else torch.device("cuda"))
        m = cls(linear.in_features, linear.out_features, bias=linear.bias is not None,
                group=group, scheme=scheme, relu=relu, device=dev, out_dtype=out_dtype)
        return m.load_weight(linear.weight, linear.bias)

    def forward(self, x: torch.Tensor) -> torch.Tensor:
        if x.shape[-1] != self.in_features:
            raise ValueError(f"expected last dimension {self.in_features}, got {x.shape[-1]}")
        lead = x.shape[:-1]
        x2 = x.reshape(-1, self.in_features).contiguous()
        y = int4_matmul(x2, self.packed, self.scales, self.in_features, self.group,
                        zeros=self.zeros, bias=self.bias, relu=self.relu)
        out_dtype = self.out_dtype if self.out_dtype is not None else x.dtype
        return y.reshape(*lead, self.out_features).to(out_dtype)

    def extra_repr(self) -> str:
        return (f"in_features={self.in_features}, out_features={self.out_features}, "
                f"bias={self.bias is not None}, group={self.group}, scheme={self.scheme}, "
                f"relu={self.relu}")


def quantize_int4_affine_into(w, group, packed, scales, zeros):
    """quantize_int4_affine writing into existing buffers (same shapes)."""
    p, s, z, _ = quantize_int4_affine(w, group)
    packed.copy_(p)
    scales.copy_(s)
    zeros.copy_(z)
