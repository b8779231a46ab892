"""fp64 CPU oracle for exact scaled-dot-product attention.

TEST INFRASTRUCTURE ONLY.  The test-suite, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` are the only callers.  The CUDA
library never imports, links or calls anything here, and nothing here imports
the CUDA library: the two sides meet only in the tests, on inputs made by
``exact_io_aware_73_b200.workloads``.

Source cited as [MM]: the marketmaker.cc blog post (Indonesian edition)
"Apakah Konteks Sehari Penuh Mengalahkan Konteks Sepuluh Menit? Perhatian
Kilat dan Pertanyaan Panjang Urutan", by section heading.  Every function is
pinned by ``tests/test_oracle_pins.py`` against closed forms, invariants,
brute force and a hand-worked fixture (``tests/golden/``).
"""
from .oracle import (  # noqa: F401
    attention,
    attention_backward,
    attention_blocked,
    attention_rows_bf16,
    attention_full_bf16,
    attention_block_sparse_rows_bf16,
    attention_block_sparse_bf16,
    attend_scores,
    softmax_row,
    bf16_bits,
    bf16_bits_to_f64,
    max_threads,
    library_path,
    e4m3_encode,
    e4m3_decode,
    hadamard_rotate,
    fp8_quantize,
    attention_fp8,
    attention_fp8_rows,
    FP8_KERNEL_TAU,
    quantize_qkv_fp8,
    attention_decode,
    attention_decode_rows_bf16,
    attention_backward_rows_bf16,
)
