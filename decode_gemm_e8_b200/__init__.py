"""E8 lattice-codebook weights decoded on the GPU and fed into a bf16 GEMM (B200, sm_100a)."""
