"""libw4a16: group-wise INT4 weight-only quantisation and the W4A16 matmul on B200."""
