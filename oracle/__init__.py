"""CPU oracle for the DiT block (test infrastructure; see dit_block.py)."""
