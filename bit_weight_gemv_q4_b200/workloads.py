"""Tensor shapes of the single-user decode workloads.

A dense ~27B hybrid model with 64 layers, 16 of them gated attention and 48
Gated DeltaNet (wiselychen guide "Qwen3.8-27B measured ...", section "Before
deploying: weights, KV cache, memory bandwidth"), hidden size 5120, FFN width
17408, grouped k/v width 1024, vocabulary 248320; the attention projections
and the output head are raised to 8 bits while the rest stays at 4 bits
(bs178.com llamAmpere post, "Why it is this fast", part two).  The pages do not
give the DeltaNet projection shapes; every mixer here uses the q/k/v/o shapes
of the attention layers, and layer i is an attention layer when i % 4 == 3.
The draft head's vocabulary map keeps 65536 of the 248320 tokens (bs178.com
post, part four).

Algorithmic weight bytes per tensor: N*K/2 + 2*N*K/32 (q4) and
N*K + 2*N*K/32 (q8): the integer codes plus one fp16 scale per group of 32.
"""
from __future__ import annotations

from dataclasses import dataclass

HIDDEN = 5120
FFN = 17408
KV = 1024
VOCAB = 248320
DRAFT_VOCAB = 65536
N_LAYERS = 64


def weight_bytes(bits: int, N: int, K: int) -> int:
    """Algorithmic bytes of one N x K group-32 tensor (codes + fp16 scales)."""
    codes = N * K // 2 if bits == 4 else N * K
    return codes + 2 * N * (K // 32)


@dataclass(frozen=True)
class Tensor:
    name: str
    bits: int
    N: int
    K: int
    tensor_id: int  # selects the generator streams

    @property
    def bytes(self) -> int:
        return weight_bytes(self.bits, self.N, self.K)


def is_attention_layer(layer: int) -> bool:
    return layer % 4 == 3


def _layer_tensors(layer: int, mixer_bits: int, fused: bool) -> list[Tensor]:
    base = 16 + 16 * layer
    if fused:
        return [
            Tensor(f"L{layer}.qkv", mixer_bits, HIDDEN + 2 * KV, HIDDEN, base + 7),
            Tensor(f"L{layer}.o", mixer_bits, HIDDEN, HIDDEN, base + 3),
            Tensor(f"L{layer}.gate_up", 4, 2 * FFN, HIDDEN, base + 8),
            Tensor(f"L{layer}.down", 4, HIDDEN, FFN, base + 6),
        ]
    return [
        Tensor(f"L{layer}.q", mixer_bits, HIDDEN, HIDDEN, base + 0),
        Tensor(f"L{layer}.k", mixer_bits, KV, HIDDEN, base + 1),
        Tensor(f"L{layer}.v", mixer_bits, KV, HIDDEN, base + 2),
        Tensor(f"L{layer}.o", mixer_bits, HIDDEN, HIDDEN, base + 3),
        Tensor(f"L{layer}.gate", 4, FFN, HIDDEN, base + 4),
        Tensor(f"L{layer}.up", 4, FFN, HIDDEN, base + 5),
        Tensor(f"L{layer}.down", 4, HIDDEN, FFN, base + 6),
    ]


def single_q4() -> list[Tensor]:
    """One q4 4096 x 4096 product (M = 1)."""
    return [Tensor("w4096", 4, 4096, 4096, 1)]


def layer_q4() -> list[Tensor]:
    """One 27B-shaped layer, every projection q4 (used at M = 1 and M = 4)."""
    return _layer_tensors(0, 4, fused=False)


def draft_heads() -> list[Tensor]:
    """The q8 vocabulary projection, mapped (65536 rows) and full (248320 rows)."""
    return [Tensor("head.mapped", 8, DRAFT_VOCAB, HIDDEN, 1022), Tensor("head.full", 8, VOCAB, HIDDEN, 1023)]


def decode_stream(fused: bool = True) -> list[Tensor]:
    """The 64-layer weight stream of one decode step plus the q8 output head,
    in execution order.  fused=True concatenates the products that share an
    input (q|k|v and gate|up), 4 products per layer; fused=False lists all 7."""
    out: list[Tensor] = []
    for layer in range(N_LAYERS):
        out += _layer_tensors(layer, 8 if is_attention_layer(layer) else 4, fused)
    out.append(Tensor("head", 8, VOCAB, HIDDEN, 1023))
    return out


def total_bytes(tensors: list[Tensor]) -> int:
    return sum(t.bytes for t in tensors)


def distinct_k(tensors: list[Tensor]) -> list[int]:
    return sorted({t.K for t in tensors})


def activation_stream_id(K: int) -> int:
    """Generator stream of the activations that feed every product with this K."""
    return K


class DeviceStream:
    """A list of products generated, packed and captured on the current CUDA
    device: the weights of every tensor (generated on the device from the
    seeded generator, then repacked by the library's device packer), one
    activation block per distinct K, one output per tensor, and the captured
    layer stack.  The oracle regenerates any row on the host from the same
    (seed, tensor id)."""

    def __init__(self, tensors: list[Tensor], M: int, seed: int = 0, flags: int = 0):
        import torch

        import bit_weight_gemv_q4_b200 as q4

        from . import synth

        self.tensors = list(tensors)
        self.M = M
        self.seed = seed
        dev = torch.device("cuda")
        max_canon = max((t.N * (t.K // 2 if t.bits == 4 else t.K) for t in self.tensors), default=0)
        max_scales = max((t.N * (t.K // 32) for t in self.tensors), default=0)
        canon = torch.empty(max(max_canon, 16), dtype=torch.uint8, device=dev)
        scales = torch.empty(max(max_scales, 8), dtype=torch.int16, device=dev)
        self.packed = []
        for t in self.tensors:
            nq = t.N * (t.K // 2 if t.bits == 4 else t.K)
            ns = t.N * (t.K // 32)
            synth.weights_device(t.bits, seed, synth.weight_stream(t.tensor_id), t.K, 0, t.N, canon[:nq])
            synth.scales_device(seed, synth.scale_stream(t.tensor_id), t.K, 0, t.N, scales[:ns])
            p = torch.empty(q4.q4_packed_bytes(t.bits, t.N, t.K), dtype=torch.uint8, device=dev)
            q4.q4_pack_weights_device(t.bits, canon[:nq], scales[:ns], t.N, t.K, p)
            self.packed.append(p)
        del canon, scales
        self.x = {}
        for K in distinct_k(self.tensors):
            xb = torch.empty(M * K, dtype=torch.int16, device=dev)
            synth.activations_device(seed, synth.act_stream(activation_stream_id(K)), M, K, xb)
            self.x[K] = xb
        self.y = [torch.empty(M * t.N, dtype=torch.float32, device=dev) for t in self.tensors]
        torch.cuda.synchronize()
        self.stack = self.make_stack(flags)

    def make_stack(self, flags: int = 0):
        """Another layer stack over the same device buffers (e.g. another mode)."""
        import bit_weight_gemv_q4_b200 as q4

        entries = [(t.bits, t.N, t.K, p, self.x[t.K], y) for t, p, y in zip(self.tensors, self.packed, self.y)]
        return q4.layer_stack_create(entries, self.M, flags)

    @property
    def weight_bytes(self) -> int:
        return total_bytes(self.tensors)

    def run(self, stream=None) -> None:
        import bit_weight_gemv_q4_b200 as q4

        q4.layer_stack_run(self.stack, stream)

    def check(self, stream=None) -> None:
        import bit_weight_gemv_q4_b200 as q4

        q4.layer_stack_check(self.stack, stream)

    def close(self) -> None:
        self.stack.close()
        self.packed.clear()
        self.y.clear()
        self.x.clear()
