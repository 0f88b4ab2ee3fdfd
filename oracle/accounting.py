"""Cache byte accounting (oracle).

Entry sizes and per-token cache growth as the DeepSeek-V4.1-Flash architecture
database states them (storage components of the cache groups, and the KV
bytes-per-token facts):

* main KV entry: 512 E2M1 elements + 32 E4M3 scales      = 256 + 32 = 288 B
* indexer-K entry: 128 E2M1 elements + 4 E8M0 scales     =  64 +  4 =  68 B
* SWA window entry: 512 E4M3 elements + 16 E8M0 scales   = 512 + 16 = 528 B
* global growth: (1/2 + 1) entries per token over the three m=2 encoder
  owners and the one m=1 decoder owner -> (3/2 + 1) * (288 + 68) = 890 B/token
  (also the DeepSeek-V4.1 blog's CSA2 paragraph: 890 bytes per token);
* uniform-BF16 payload accounting: 3,200 B/token global; 3,240 B/token and
  424,673,280 B per sequence at 131,072 tokens including 40 SWA windows.
"""
from __future__ import annotations

from fractions import Fraction


def entry_bytes(elements: int, elem_bits: int, block: int, scale_bits: int = 8) -> int:
    """Bytes of one entry: packed elements plus one scale per block."""
    assert (elements * elem_bits) % 8 == 0 and elements % block == 0
    return elements * elem_bits // 8 + (elements // block) * scale_bits // 8


MAIN_KV_BYTES = entry_bytes(512, 4, 16)      # 288
INDEXER_K_BYTES = entry_bytes(128, 4, 32)    # 68
SWA_BYTES = entry_bytes(512, 8, 32)          # 528


def global_bytes_per_token(groups) -> Fraction:
    """Sum over cache groups of n_owner_layers * bytes_per_entry / tokens_per_entry."""
    return sum((Fraction(n * b, m) for n, b, m in groups), Fraction(0))


def v41_flash_groups(main_bytes: int, idx_bytes: int):
    """(owners, bytes/entry, tokens/entry): 3 encoder owners at m=2, 1 decoder owner at m=1."""
    return [(3, main_bytes, 2), (3, idx_bytes, 2), (1, main_bytes, 1), (1, idx_bytes, 1)]


def retained_bytes(T: int, groups, swa_layers: int, swa_bytes: int, window: int) -> int:
    """Per-sequence retained cache: floor(T/m) entries per group plus the SWA rings."""
    total = sum(n * b * (T // m) for n, b, m in groups)
    return total + swa_layers * swa_bytes * min(T, window)
