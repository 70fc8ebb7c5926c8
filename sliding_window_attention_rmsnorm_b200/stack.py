"""Per-layer driver of the attention core for an "SSSL" layer stack.

The window of each layer comes from the library (ar_attn_layer_window): the
pattern repeats over layers, 'S' is half the sequence length, 'L' the full
length, and the last layer is always global ("autoresearch" README on gitee,
section 5.2.2; web3.okx.com review, paragraph on the SSSL pattern).  Layers here
take independent inputs, as in the stacked workloads this core is measured on.
"""
from . import attn


def layer_windows(n_layer: int, seq_len: int, pattern: str = "SSSL"):
    out = []
    for layer in range(n_layer):
        w = attn.lib().ar_attn_layer_window(layer, n_layer, seq_len, pattern.encode())
        if w < 0:
            raise ValueError("invalid window pattern %r" % pattern)
        out.append(w)
    return out


def ve_layers(n_layer: int):
    """Layers that mix in a value embedding: every other layer, the last one
    included ("autoresearch" README (gitee), section 5.2.3)."""
    return [l for l in range(n_layer) if l % 2 == (n_layer - 1) % 2]


class Stack:
    """Forward and backward of every layer, enqueued back to back on one stream.

    layers: list of dicts with bf16 CUDA tensors q, dO [B, T, H, 128] and k, v
    [B, T, Hkv, 128] (Hkv = H, or fewer for grouped K/V heads), and, on layers
    with a value embedding, ve [B, T, Hkv, 128] and g [B, T, Hkv].
    rope: optional (cos, sin) tables; with them every layer runs the fused RoPE
    path (fwd_rope / bwd_rope), with the value embedding where a layer has one.
    Outputs (o, lse, dq, dk, dv[, dve, dg]) and scratch are allocated once and reused;
    with rope, each layer's forward workspace (its rotated k and mixed v) is kept
    for that layer's backward, which then rotates only q.
    """

    def __init__(self, layers, pattern: str = "SSSL", eps: float = 1e-6, scale=None, windows=None, rope=None):
        import torch
        self.layers = layers
        B, T, H, D = layers[0]["q"].shape
        Hkv = layers[0]["k"].shape[2]
        self.windows = list(windows) if windows is not None else layer_windows(len(layers), T, pattern)
        self.eps, self.scale = eps, scale
        dev = layers[0]["q"].device
        self.out = [dict(o=torch.empty_like(L["q"]),
                         lse=torch.empty((B, H, T), dtype=torch.float32, device=dev),
                         dq=torch.empty_like(L["q"]), dk=torch.empty_like(L["k"]),
                         dv=torch.empty_like(L["v"])) for L in layers]
        self.rope = rope
        if rope is None:
            self.ws_bwd = torch.empty(attn.bwd_workspace_bytes(B, T, H, D, Hkv), dtype=torch.uint8, device=dev)
        else:
            with_ve = any("ve" in L for L in layers)
            self.ws_bwd = torch.empty(attn.bwd_rope_workspace_bytes(B, T, H, D, Hkv, with_ve), dtype=torch.uint8,
                                      device=dev)
            # each layer's forward pre-pass output (rotated k, mixed v) is kept, as
            # an activation, for that layer's backward
            self.ws_fwd = [torch.empty(attn.fwd_rope_workspace_bytes(B, T, Hkv, D, "ve" in L), dtype=torch.uint8,
                                       device=dev) for L in layers]
            for L, O in zip(layers, self.out):
                if "ve" in L:
                    O["dve"] = torch.empty_like(L["ve"])
                    O["dg"] = torch.empty((B, T, Hkv), dtype=torch.float32, device=dev)

    def forward_layer(self, l: int):
        L, O, w = self.layers[l], self.out[l], self.windows[l]
        if self.rope is None:
            attn.fwd(L["q"], L["k"], L["v"], w, self.eps, self.scale, out=O["o"], lse=O["lse"])
        else:
            attn.fwd_rope(L["q"], L["k"], L["v"], self.rope[0], self.rope[1], w, self.eps, self.scale,
                          ve=L.get("ve"), ve_gate=L.get("g"), out=O["o"], lse=O["lse"], workspace=self.ws_fwd[l])

    def backward_layer(self, l: int):
        L, O, w = self.layers[l], self.out[l], self.windows[l]
        if self.rope is None:
            attn.bwd(L["q"], L["k"], L["v"], O["o"], L["dO"], O["lse"], w, self.eps, self.scale,
                     dq=O["dq"], dk=O["dk"], dv=O["dv"], workspace=self.ws_bwd)
        else:
            attn.bwd_rope(L["q"], L["k"], L["v"], O["o"], L["dO"], O["lse"], self.rope[0], self.rope[1], w,
                          self.eps, self.scale, ve=L.get("ve"), ve_gate=L.get("g"), dq=O["dq"], dk=O["dk"],
                          dv=O["dv"], dve=O.get("dve"), dgate=O.get("dg"), workspace=self.ws_bwd,
                          saved=self.ws_fwd[l])

    def forward(self):
        for l in range(len(self.layers)):
            self.forward_layer(l)

    def backward(self):
        for l in reversed(range(len(self.layers))):
            self.backward_layer(l)

    def step(self):
        self.forward()
        self.backward()
