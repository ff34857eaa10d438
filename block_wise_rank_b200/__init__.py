"""B200-native MILO block-wise low-rank KV compression (libmilo binding)."""
