"""A synthetic model laid out in device (and pinned host) memory.

Benchmark and test infrastructure: allocates, with torch, every buffer a
decode engine needs -- one canonical blob per layer (device memory, or pinned
host memory for host-tier layers), the fp16 embedding table, the final norm,
the output head, per-layer fp16 KV caches holding the prior context, the two
device slots -- and fills them from the seeded generator (its CUDA twin for
full-size models, or the host build uploaded for small ones).  It knows nothing
of the method's arithmetic and does not call the library under test.
"""
from __future__ import annotations

import numpy as np

from . import BLOCK_BYTES, BLOCK_ELEMS, dev_fill_f16, dev_fill_f32, dev_quant_rows, fill_f16, fill_f32, quant_rows
from . import workloads as wl


class DeviceModel:
    def __init__(self, d: dict, qtype: int, head_qtype: int, sd: int, max_ctx: int, n_prior: int,
                 tier_map=None, source: str = "device", keep_resident_copy: bool = False):
        import torch
        self.torch = torch
        self.d, self.qtype, self.head_qtype, self.sd = d, qtype, head_qtype, sd
        self.max_ctx, self.n_prior = max_ctx, n_prior
        L, H, V = d["n_layers"], d["hidden"], d["vocab"]
        self.tier_map = list(tier_map) if tier_map is not None else [0] * L
        self.blob_bytes, self.offsets = wl.layer_layout(d, qtype)
        cuda = torch.device("cuda")
        host_src = source == "host"

        def dev_u8(n):
            return torch.zeros(n, dtype=torch.uint8, device=cuda)

        self.layers = []            # blob actually used (device or pinned host)
        self.resident_copy = []     # device blob for every layer when keep_resident_copy
        for l in range(L):
            blob = dev_u8(self.blob_bytes)
            if host_src:
                hb, _ = wl.host_layer_blob(d, qtype, sd, l)
                blob.copy_(torch.from_numpy(hb))
            else:
                wl.dev_layer_blob(d, qtype, sd, l, blob.data_ptr())
            if self.tier_map[l] == 1:
                torch.cuda.synchronize()
                hostb = torch.empty(self.blob_bytes, dtype=torch.uint8, pin_memory=True)
                hostb.copy_(blob)
                self.layers.append(hostb)
                if keep_resident_copy:
                    self.resident_copy.append(blob)
                else:
                    del blob
            else:
                self.layers.append(blob)
                self.resident_copy.append(blob)
        n_emb = V * H
        self.embed = torch.empty(n_emb, dtype=torch.int16, device=cuda)
        self.final_norm = torch.empty(H, dtype=torch.float32, device=cuda)
        rb = H // BLOCK_ELEMS[head_qtype] * BLOCK_BYTES[head_qtype]
        self.head = dev_u8(V * rb)
        if host_src:
            self.embed.copy_(torch.from_numpy(fill_f16(sd, "embed", n_emb, 0.0, wl.EMB_SIGMA).view(np.int16)))
            self.final_norm.copy_(torch.from_numpy(fill_f32(sd, "final_norm", H, 1.0, wl.NORM_SIGMA)))
            self.head.copy_(torch.from_numpy(quant_rows(head_qtype, sd, "head", V, H, sigma=wl.W_SIGMA).ravel()))
        else:
            dev_fill_f16(sd, "embed", n_emb, 0.0, wl.EMB_SIGMA, self.embed.data_ptr())
            dev_fill_f32(sd, "final_norm", H, 1.0, wl.NORM_SIGMA, self.final_norm.data_ptr())
            dev_quant_rows(head_qtype, sd, "head", V, H, self.head.data_ptr(), sigma=wl.W_SIGMA)
        Hkv, D = d["n_kv_heads"], d["head_dim"]
        self.k_caches, self.v_caches = [], []
        for l in range(L):
            k = torch.zeros(Hkv * max_ctx * D, dtype=torch.int16, device=cuda)
            v = torch.zeros_like(k)
            self.k_caches.append(k)
            self.v_caches.append(v)
        self.reset_kv()
        any_host = any(t == 1 for t in self.tier_map)
        self.slots = [dev_u8(self.blob_bytes), dev_u8(self.blob_bytes)] if any_host else [None, None]
        torch.cuda.synchronize()

    def reset_kv(self):
        """Caches back to the prior context: rows < n_prior from the prior stream, the rest 0."""
        torch = self.torch
        d, L = self.d, self.d["n_layers"]
        for l in range(L):
            k, v = self.host_kv(l)
            self.k_caches[l].copy_(torch.from_numpy(k.view(np.int16).ravel()))
            self.v_caches[l].copy_(torch.from_numpy(v.view(np.int16).ravel()))

    def host_kv(self, l):
        return wl.host_kv_prior(self.d, self.sd, l, self.max_ctx, self.n_prior)

    # ----------------------------------------------------------- host views
    def host_layer_tensors(self, l: int) -> dict:
        """The layer's tensors as numpy arrays copied back from where the model
        holds them (for the oracle); equal to the generator's host output."""
        blob = self.layers[l]
        b = blob.cpu().numpy() if blob.is_cuda else blob.numpy()
        return wl.tensors_from_blob(b, self.d, self.qtype)

    def host_embed(self):
        return self.embed.cpu().numpy().view(np.uint16)

    def host_final_norm(self):
        return self.final_norm.cpu().numpy()

    def host_head(self):
        V = self.d["vocab"]
        return self.head.cpu().numpy().reshape(V, -1)

    def weight_bytes_per_token(self, n_ctx: int, layers: int | None = None) -> int:
        return wl.bytes_per_token(self.d, self.qtype, self.head_qtype, n_ctx, layers)
