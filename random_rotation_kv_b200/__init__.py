"""random_rotation_kv_b200 — random-rotation KV / embedding vector quantisation on B200."""
