"""One decode step of a small batch through the library's step runtime.

    python examples/decode_step.py

Shapes as in include/pa.h: caches [num_blocks, num_kv_heads, block_size, head_dim],
q / out [S, num_heads, head_dim], the new tokens' K/V rows [S, num_kv_heads, head_dim].
"""
import math
import os
import sys

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import torch  # noqa: E402

from paged_kv_cache_342_b200.runtime import PagedDecoder  # noqa: E402

NB, Hkv, bs, D, Hq = 8192, 8, 16, 128, 64
k_cache = torch.zeros(NB, Hkv, bs, D, dtype=torch.bfloat16, device="cuda")
v_cache = torch.zeros_like(k_cache)
dec = PagedDecoder(k_cache, v_cache, num_heads=Hq, scale=1 / math.sqrt(D),
                   max_blocks_per_seq=256)
for sid, n in enumerate([700, 1200, 35]):
    dec.admit(sid, n)                    # block manager: ceil(n / bs) blocks each
dec.bind([0, 1, 2])                      # the batch; its device buffers come from torch
q = torch.randn(3, Hq, D, dtype=torch.bfloat16, device="cuda")
new_k = torch.randn(3, Hkv, D, dtype=torch.bfloat16, device="cuda")
new_v = torch.randn_like(new_k)
out = torch.empty_like(q)
info = dec.step(q, new_k, new_v, out)    # append slots, copy-on-write, cache write, attention

if __name__ == "__main__":
    torch.cuda.synchronize()
    print("sequence lengths after the step:", info.lens.tolist())
