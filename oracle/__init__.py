"""CPU oracle for PACK3D attention (float64). Test infrastructure: see pack3d_oracle.py."""
